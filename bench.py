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
ROTATE_BYTES = 3 * (126 << 20)  # consecutive steps' inputs span more than 3x the L2
MAX_REPLICAS = 64
# tokens per page of the paged caches (the fixed token-block size a neighbouring page's
# hardware-efficiency section gives as its example)
PAGE_SIZE = 128
PEAKS_FILE = os.path.join(ROOT, "MEASURED_PEAKS.json")
TRAFFIC_FILE = os.path.join(ROOT, "profiles", "traffic.json")
FALLBACK_HBM_GBS = 6650.0


# ----------------------------------------------------------------------------- helpers

def _dist_env():
    ws = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return ws, rank, local


def rank_seed(base: int, rank: int) -> int:
    """Each rank decodes its own independent sequences (weak scaling: the (sequence, KV head)
    units shard with no exchange), drawn from a rank-specific seed."""
    return base + 7919 * rank


def reduce_over_ranks(values, device=None):
    """Per-rank timings -> their maximum over the ranks (the job ends with its slowest rank);
    the identity without a process group."""
    if not torch.distributed.is_available() or not torch.distributed.is_initialized() \
            or torch.distributed.get_world_size() == 1:
        return [float(v) for v in values]
    t = torch.tensor([float(v) for v in values], device=device, dtype=torch.float64)
    torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
    return [float(x) for x in t.tolist()]


def job_tokens_per_s(tokens_per_rank_step: int, world: int, ms_per_step: float) -> float:
    """Whole-job throughput: the tokens every rank decodes per step over the slowest rank's
    step time."""
    return tokens_per_rank_step * world / (ms_per_step / 1e3)


def _hbm_peak():
    try:
        with open(PEAKS_FILE) as f:
            p = json.load(f)
        return float(p["hbm_gbs"]), "measured"
    except Exception:
        return FALLBACK_HBM_GBS, "fallback"


def _kernel_source_hash() -> str:
    """Hash of the decode kernel's device code (the kernel template and its device helpers)."""
    h = hashlib.sha256()
    for name in ("decode_kernel.cuh", "stief_device.cuh"):
        h.update(open(os.path.join(ROOT, "decode_attention_stief_b200", "csrc", name), "rb").read())
    return h.hexdigest()[:16]


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
    """Per-layer caches with room for w.L + total_steps tokens."""
    import decode_attention_stief_b200 as stief
    L_max = w.L + total_steps + 1
    layers = []
    for li, (rK, rV) in enumerate(w.layer_ranks()):
        lay = Layer(w, li, rK, rV, w.L - 1, L_max, seed, dev)
        lay.ws = stief.workspace_for(w.B, w.Hq, w.Hkv, rV, L_max, device=dev)
        layers.append(lay)
    return layers, L_max


def _int4(args) -> bool:
    """The 4-bit form of the int8 mode (argument namespaces built elsewhere may lack the flag)."""
    return bool(getattr(args, "int4", False))


def step_call(args) -> str:
    """The API call whose kernel a step of the chosen mode runs (one per layer)."""
    if args.int8:
        return "stief_decode_attention_q4" if _int4(args) else "stief_decode_attention_q8"
    if args.joint:
        return "stief_decode_latent_joint_v" if args.latent else "stief_decode_attention_joint_v"
    if args.latent:
        return "stief_decode_latent"
    if args.paged:
        return "stief_append_decode_paged"
    return "stief_decode_attention" if args.unfused else "stief_append_decode"


def row_bytes_fn(w: si.Workload, int8: bool = False, joint: bool = False, int4: bool = False):
    """Cache bytes per (token, sequence, KV head) for a layer of ranks (rK, rV): bf16 rows, int8
    or 4-bit rows with their two fp32 scales, or per-head keys with one joint value row shared
    by the Hkv heads (its bytes split over them)."""
    if int4:
        return lambda rK, rV: (rK + rV) // 2 + 8
    if int8:
        return lambda rK, rV: rK + rV + 8
    if joint:
        return lambda rK, rV: 2 * rK + 2 * rV / w.Hkv
    return lambda rK, rV: 2 * (rK + rV)


def replica_count(w: si.Workload, int8: bool = False, joint: bool = False, int4: bool = False) -> int:
    """Copies of the workload's layer state that consecutive timed steps rotate over, so that
    the inputs of a step were last touched at least ROTATE_BYTES of cache reads earlier
    (more than 3x the 126 MB L2: every step streams its cache from HBM, and no flush is
    needed between steps)."""
    rb = row_bytes_fn(w, int8, joint, int4)
    per = int(sum(rb(rK, rV) * w.B * w.Hkv * w.L for rK, rV in w.layer_ranks()))
    return 1 if per >= ROTATE_BYTES else min(MAX_REPLICAS, -(-ROTATE_BYTES // per))


def step_description(args) -> str:
    """What one timed step runs, in words (the same text in both arms)."""
    if args.int8:
        what = (("decode over a 4-bit latent cache (two codes per byte + fp32 row scales"
                 if _int4(args) else "decode over an int8 latent cache (codes + fp32 row scales")
                + ", synthetic values), no append, every layer; ")
    elif args.joint:
        what = ("decode with per-head keys and one joint value latent per token shared by the "
                "KV heads" + (" (latent output)" if args.latent else "") + ", no append, every "
                "layer; ")
    elif args.latent:
        what = ("latent decode only (bases folded into the attention weights: q~ in, o~ out; the "
                "new token's latent rows would come from the folded K/V projection), every "
                "layer; ")
    elif args.paged:
        what = (f"append 1 token per (sequence, KV head) + decode over page pools ({PAGE_SIZE}-"
                f"token pages at shuffled pool positions), every layer; ")
    else:
        what = "append 1 token per (sequence, KV head) + decode, every layer; "
    how = ("the API calls captured in CUDA graphs (one step per replica, the timed region "
           "replays the replica cycle back to back); ")
    calls = ("stief_compress_append + stief_decode_attention (3 kernels per layer)"
             if args.unfused else f"{step_call(args)} (1 kernel per layer)")
    return what + how + calls


def config_dict(w: si.Workload, args, world: int) -> dict:
    """The workload and how it is run: identical in the GPU arm and the reference arm."""
    R = replica_count(w, args.int8, args.joint, _int4(args))
    rb = row_bytes_fn(w, args.int8, args.joint, _int4(args))
    rot_mb = R * sum(rb(rK, rV) * w.B * w.Hkv * w.L for rK, rV in w.layer_ranks()) / 2**20
    appends = not (args.latent or args.int8 or args.joint)
    ranks = [list(r) for r in w.layer_ranks()]
    return {
        "workload": w.name, "B": w.B, "Hq": w.Hq, "Hkv": w.Hkv, "d": w.d, "context": w.L,
        "layers": len(ranks), "ranks": ranks[:4] + (["..."] if len(ranks) > 4 else []),
        "step": step_description(args),
        "context_growth": (f"+1 token per step of a replica, from context {w.L}" if appends
                           else f"none (context {w.L} every step)"),
        "l2": (f"no flush: steps rotate over {R} copies of the layer caches ({rot_mb:.0f} MiB in "
               f"all, > 3x the 126 MB L2)" if R > 1 else
               f"no flush: one step reads {rot_mb:.0f} MiB of caches (> 3x the 126 MB L2)"
               if rot_mb * 2**20 >= ROTATE_BYTES else
               f"inputs ({rot_mb:.1f} MiB in {R} copies) fit in L2: a latency case"),
        "parallelism": f"independent sequences per GPU x{world}",
    }


def to_pages(cache: torch.Tensor, page_size: int, perm: torch.Tensor):
    """A contiguous latent cache [B][Hkv][L][r] as a page pool and block table.

    Page j of sequence b (its tokens [j*page_size, (j+1)*page_size), every KV head) goes to
    pool entry perm[b*max_pages + j]; the cache is zero-padded to whole pages.  Returns
    (pool [B*max_pages][Hkv][page_size][r], block_table [B][max_pages] int32).
    """
    B, Hkv, L, r = cache.shape
    mp = -(-L // page_size)
    if mp * page_size != L:
        cache = torch.nn.functional.pad(cache, (0, 0, 0, mp * page_size - L))
    blocks = cache.reshape(B, Hkv, mp, page_size, r).permute(0, 2, 1, 3, 4)
    pool = torch.empty((B * mp, Hkv, page_size, r), dtype=cache.dtype, device=cache.device)
    pool[perm.to(cache.device)] = blocks.reshape(B * mp, Hkv, page_size, r)
    return pool, perm.reshape(B, mp).to(device=cache.device, dtype=torch.int32)


def _backlog():
    """Queue ~50 us of GPU work so the events that follow are not exposed to host launch gaps."""
    torch.cuda._sleep(100000)


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
    seed = rank_seed(w.seed, rank)
    W, K = args.warmup, args.steps
    R = replica_count(w, args.int8, args.joint, _int4(args))
    reps = []
    for r in range(R):
        # room for every append of the warm-up, timed and kernel-timing runs of a replica
        layers, L_max = build_state(w, W + K + 2 * args.decode_iters + 64, seed + 104729 * r, dev)
        reps.append(layers)
    layers = reps[0]
    g = torch.Generator(device=dev)
    g.manual_seed(seed + 1)
    # The step's inputs live in one device staging buffer, filled by one H2D copy per step in
    # the end-to-end timing: q [B][Hq][d], then the new token's k and v rows [B][Hkv][1][d]
    # (latent mode: q~ [B][Hq][r_K] of every layer, one after the other).  Every view starts
    # on a 32-byte boundary.
    if args.latent:
        sizes = [w.B * w.Hq * lay.rK for lay in layers]
    else:
        sizes = [w.B * w.Hq * w.d, w.B * w.Hkv * w.d, w.B * w.Hkv * w.d]
    inp = torch.randn((sum(sizes),), generator=g, device=dev).to(torch.bfloat16)
    views = list(torch.split(inp, sizes))
    if args.latent:
        qlat_s = [v.view(w.B, w.Hq, lay.rK) for v, lay in zip(views, layers)]
        q_s = k_s = v_s = None
    else:
        qlat_s = []
        q_s = views[0].view(w.B, w.Hq, w.d)
        k_s = views[1].view(w.B, w.Hkv, 1, w.d)
        v_s = views[2].view(w.B, w.Hkv, 1, w.d)
    out = torch.empty((len(layers), w.B, w.Hq, w.d), dtype=torch.bfloat16, device=dev)
    status = torch.zeros(1, dtype=torch.int32, device=dev)
    # int8 mode: every replica's layer caches as int8 codes and fp32 row scales (synthetic:
    # the decode's cost does not depend on the values); L_max a multiple of 64
    if args.int8:
        for lays in reps:
            for lay in lays:
                L8 = (L_max + 63) // 64 * 64
                if _int4(args):  # two 4-bit codes per byte: any byte is a valid pair
                    lay.kq = torch.randint(0, 256, (w.B, w.Hkv, L8, lay.rK // 2), generator=g,
                                           device=dev, dtype=torch.uint8)
                    lay.vq = torch.randint(0, 256, (w.B, w.Hkv, L8, lay.rV // 2), generator=g,
                                           device=dev, dtype=torch.uint8)
                else:
                    lay.kq = torch.randint(-127, 128, (w.B, w.Hkv, L8, lay.rK), generator=g,
                                           device=dev, dtype=torch.int8)
                    lay.vq = torch.randint(-127, 128, (w.B, w.Hkv, L8, lay.rV), generator=g,
                                           device=dev, dtype=torch.int8)
                lay.ks = torch.rand((w.B, w.Hkv, L8), generator=g, device=dev) * 0.02
                lay.vs = torch.rand((w.B, w.Hkv, L8), generator=g, device=dev) * 0.02
                lay.k_lat = lay.v_lat = None  # the bf16 caches are not used
    # paged mode: every replica's layer caches moved into pools of PAGE_SIZE-token pages, the
    # pages of each sequence at shuffled pool positions (one block table per layer)
    if args.paged:
        gp = torch.Generator()
        gp.manual_seed(seed + 2)
        for lays in reps:
            for lay in lays:
                perm = torch.randperm(w.B * -(-L_max // PAGE_SIZE), generator=gp)
                lay.k_pages, lay.block_table = to_pages(lay.k_lat, PAGE_SIZE, perm)
                lay.v_pages, _ = to_pages(lay.v_lat, PAGE_SIZE, perm)
                lay.k_lat = lay.v_lat = None  # the contiguous caches are not used
    # joint mode: per layer one joint value basis P_VJ [Hkv*d][rV] and one value latent per
    # token v_joint [B][L_max][rV] shared by the KV heads (the per-head value caches dropped)
    if args.joint:
        for ri, lays in enumerate(reps):
            for li, lay in enumerate(lays):
                js = si.sub_seed(seed, 14, li, ri)
                lay.P_VJ = si.to_bf16(si.bases(js, 1, w.Hkv * w.d, lay.rV)[0]).to(dev)
                lay.v_joint = si.latent_cache_torch(js, w.B, 1, L_max, lay.rV, 1, dev)[:, 0]
                lay.v_joint = lay.v_joint.contiguous()
                lay.v_lat = None
    # outputs: one device buffer read back by one D2H copy per step (latent mode: o~ of every
    # layer, one after the other)
    if args.latent:
        osizes = [w.B * w.Hq * lay.rV for lay in layers]
        out_all = torch.empty((sum(osizes),), dtype=torch.bfloat16, device=dev)
        olat = [v.view(w.B, w.Hq, lay.rV) for v, lay in zip(torch.split(out_all, osizes), layers)]
    else:
        out_all = out
        olat = []

    def layer_step(li, lay):
        if args.int8:  # decode over the int8 (or 4-bit) cache (no append)
            (stief.stief_decode_attention_q4 if _int4(args) else stief.stief_decode_attention_q8)(q_s, lay.P_K, lay.P_V, lay.kq, lay.vq, lay.ks, lay.vs,
                                            lay.seq_lens, out[li], lay.ws, max_seq_len=L_max,
                                            num_splits=args.splits, dev_status=status)
        elif args.latent and args.joint:  # latent output over the joint value latent
            stief.stief_decode_latent_joint_v(qlat_s[li], lay.k_lat, lay.v_joint, lay.seq_lens,
                                              olat[li], lay.ws, max_seq_len=L_max,
                                              num_splits=args.splits, dev_status=status)
        elif args.latent:  # attention in the latent space only (no projections, no append)
            stief.stief_decode_latent(qlat_s[li], lay.k_lat, lay.v_lat, lay.seq_lens, olat[li],
                                      lay.ws, max_seq_len=L_max, num_splits=args.splits,
                                      dev_status=status)
        elif args.joint:  # decode with per-head keys and the joint value latent (no append)
            stief.stief_decode_attention_joint_v(q_s, lay.P_K, lay.P_VJ, lay.k_lat, lay.v_joint,
                                                 lay.seq_lens, out[li], lay.ws,
                                                 max_seq_len=L_max, num_splits=args.splits,
                                                 dev_status=status)
        elif args.paged:  # append + decode in one kernel, over page pools
            stief.stief_append_decode_paged(q_s, k_s, v_s, lay.P_K, lay.P_V, lay.k_pages,
                                            lay.v_pages, lay.block_table, lay.seq_lens, out[li],
                                            lay.ws, max_seq_len=L_max, num_splits=args.splits,
                                            dev_status=status)
        elif args.unfused:  # the two separate calls (three kernels)
            stief.stief_compress_append(k_s, v_s, lay.P_K, lay.P_V, lay.k_lat, lay.v_lat,
                                        lay.seq_lens, dev_status=status)
            stief.stief_decode_attention(q_s, lay.P_K, lay.P_V, lay.k_lat, lay.v_lat,
                                         lay.seq_lens, out[li], lay.ws, max_seq_len=L_max,
                                         num_splits=args.splits, dev_status=status)
        else:  # append + decode in one kernel
            stief.stief_append_decode(q_s, k_s, v_s, lay.P_K, lay.P_V, lay.k_lat, lay.v_lat,
                                      lay.seq_lens, out[li], lay.ws, max_seq_len=L_max,
                                      num_splits=args.splits, dev_status=status)

    def step(lays):
        for li, lay in enumerate(lays):
            layer_step(li, lay)

    def decode_only(lays):
        """One launch of the step's attention kernel on layer 0 (for the kernel's own timing)."""
        lay = lays[0]
        if args.unfused and not args.latent and not args.int8:
            stief.stief_decode_attention(q_s, lay.P_K, lay.P_V, lay.k_lat, lay.v_lat,
                                         lay.seq_lens, out[0], lay.ws, max_seq_len=L_max,
                                         num_splits=args.splits, dev_status=status)
        else:
            layer_step(0, lay)

    def reset_lengths(L0):
        if args.latent or args.int8 or args.joint:  # no append: every step attends over the full context
            L0 = w.L
        for lays in reps:
            for lay in lays:
                lay.seq_lens.fill_(L0)

    def barrier():
        if ws_n > 1:
            torch.distributed.barrier()

    # ---- warm-up through the API (initialises the library's host-side caches), then one
    # CUDA graph per replica for: the step, the step with its host copies, and a run of
    # decode launches (layer 0) for the kernel's own timing
    for i in range(W):
        step(reps[i % R])
    torch.cuda.synchronize()
    h_inp = inp.cpu().pin_memory()
    h_out = torch.empty(out_all.shape, dtype=out_all.dtype).pin_memory()

    def e2e_step(lays):
        """One step as a user runs it: the inputs H2D (one copy from pinned memory), the API
        calls, the outputs D2H (one copy into pinned memory)."""
        inp.copy_(h_inp, non_blocking=True)
        step(lays)
        h_out.copy_(out_all, non_blocking=True)

    # the same step with prepared calls (stief.prepare: the binding's checks once per
    # buffer set; every step still goes through the C entry points): what a serving loop
    # that reuses its buffers runs
    try:
        prepared = [[stief.prepare(layer_step, li, lay) for li, lay in enumerate(lays)]
                    for lays in reps]
    except ValueError:  # a mode with more than one library call per layer
        prepared = None

    def e2e_step_prepared(r):
        inp.copy_(h_inp, non_blocking=True)
        for call in prepared[r]:
            call()
        h_out.copy_(out_all, non_blocking=True)
    n_dec = max(8, R) // R * R
    cap = torch.cuda.Stream(device=dev)
    cap.wait_stream(torch.cuda.current_stream())
    step_graphs, e2e_graphs = [], []
    cycle_graph = torch.cuda.CUDAGraph()  # one step on every replica in turn
    with torch.cuda.stream(cap):
        with torch.cuda.graph(cycle_graph, stream=cap):
            for r in range(R):
                step(reps[r])
        for r in range(R):
            gr = torch.cuda.CUDAGraph()
            with torch.cuda.graph(gr, stream=cap):
                step(reps[r])
            step_graphs.append(gr)
            ge = torch.cuda.CUDAGraph()
            with torch.cuda.graph(ge, stream=cap):
                e2e_step(reps[r])
            e2e_graphs.append(ge)
        dec_graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(dec_graph, stream=cap):
            for i in range(n_dec):
                decode_only(reps[i % R])
        # load for the clock samples: attention without appends (lengths stay put)
        warm_graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(warm_graph, stream=cap):
            for i in range(n_dec):
                lay = reps[i % R][0]
                if args.int8 or args.joint or args.latent:
                    layer_step(0, lay)
                elif args.paged:
                    stief.stief_decode_attention_paged(q_s, lay.P_K, lay.P_V, lay.k_pages,
                                                       lay.v_pages, lay.block_table, lay.seq_lens,
                                                       out[0], lay.ws, max_seq_len=L_max,
                                                       dev_status=status)
                else:
                    stief.stief_decode_attention(q_s, lay.P_K, lay.P_V, lay.k_lat, lay.v_lat,
                                                 lay.seq_lens, out[0], lay.ws, max_seq_len=L_max,
                                                 dev_status=status)
    torch.cuda.synchronize()
    stream = torch.cuda.current_stream()

    # ---- timed region: K steps, each one graph replay (append + decode, every layer);
    # consecutive steps use different replicas
    reset_lengths(w.L - 1 - W)
    for i in range(W):
        step_graphs[i % R].replay()
    reset_lengths(w.L - 1)
    torch.cuda.synchronize()
    t0_ev, t1_ev = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    cvd = os.environ.get("CUDA_VISIBLE_DEVICES")
    smi_id = cvd.split(",")[local].strip() if cvd else str(local)
    with ClockSampler(smi_id) as clk:
        # keep the GPU loaded (decode only, lengths unchanged) so the clock samples that
        # bracket the timed region are taken under load
        t_keep = time.perf_counter()
        while time.perf_counter() - t_keep < args.clock_window:
            for _ in range(10):
                warm_graph.replay()
            torch.cuda.synchronize()
        barrier()
        torch.cuda.synchronize()
        t_wall0 = time.perf_counter()
        _backlog()
        # exactly K steps: K // R replays of the R-step cycle, then single steps
        t0_ev.record(stream)
        for _ in range(K // R):
            cycle_graph.replay()
        for j in range(K % R):
            step_graphs[j].replay()
        t1_ev.record(stream)
        torch.cuda.synchronize()
        barrier()
        t_wall = time.perf_counter() - t_wall0
        time.sleep(0.25)  # one more sample after the timed region
    ms_per_step = t0_ev.elapsed_time(t1_ev) / K
    clocks = clk.summary()
    st = stief.stief_read_device_status(status)
    if st != 0:
        raise RuntimeError(f"device status {st:#x} after the timed steps")
    L_dec = int(reps[0][0].seq_lens[0].item())
    ctx_first, ctx_last = w.L, int(max(int(lays[0].seq_lens[0].item()) for lays in reps))

    # ---- decode kernel timing for the roofline: runs of n_dec back-to-back launches
    # (replicas rotating), averaged over the timed region; plus single launches.  The fused
    # kernel appends a token per launch: lengths restart at L_dec - 1 for each run.
    appends = not (args.unfused or args.latent or args.int8 or args.joint)  # the kernel appends
    L_run0 = L_dec - (1 if appends else 0)
    reset_lengths(L_run0)
    dec_reps = max(3, args.decode_iters // n_dec)
    torch.cuda.synchronize()
    _backlog()
    d0, d1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    d0.record(stream)
    for _ in range(dec_reps):
        dec_graph.replay()
    d1.record(stream)
    torch.cuda.synchronize()
    dec_us = d0.elapsed_time(d1) * 1e3 / (dec_reps * n_dec)
    L_dec_mean = L_dec + ((dec_reps * n_dec // R) / 2 if appends else 0)
    reset_lengths(L_run0)
    iso = []
    for j in range(max(5, min(args.decode_iters, 30))):
        _backlog()
        a0, a1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a0.record(stream)
        decode_only(reps[j % R])
        a1.record(stream)
        torch.cuda.synchronize()
        iso.append(a0.elapsed_time(a1) * 1e3)
    iso.sort()
    dec_us_iso = iso[len(iso) // 2]

    # ---- end to end through the public API, two ways, each step with one H2D copy of its
    # inputs from pinned memory and one D2H copy of its outputs into pinned memory:
    #  - api: the Python binding calls the C entry points every step (host cost included);
    #  - graph: the same calls captured once in a CUDA graph, one replay per step.
    def time_e2e(run_one):
        reset_lengths(w.L - 1 - W)
        for i in range(W):
            run_one(i)
        reset_lengths(w.L - 1)
        e0_ev, e1_ev = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        barrier()
        torch.cuda.synchronize()
        e0_ev.record(stream)
        for j in range(K):
            run_one(j)
        e1_ev.record(stream)
        torch.cuda.synchronize()
        barrier()
        return e0_ev.elapsed_time(e1_ev) / K

    e2e_plain_ms = time_e2e(lambda j: e2e_step(reps[j % R]))
    e2e_api_ms = time_e2e(lambda j: e2e_step_prepared(j % R)) if prepared is not None else e2e_plain_ms
    e2e_graph_ms = time_e2e(lambda j: e2e_graphs[j % R].replay())
    h2d = h_inp.numel() * h_inp.element_size()
    d2h = h_out.numel() * h_out.element_size()
    st = stief.stief_read_device_status(status)
    if st != 0:
        raise RuntimeError(f"device status {st:#x} after the e2e steps")

    ms_per_step, e2e_api_ms, e2e_graph_ms, dec_us, e2e_plain_ms = reduce_over_ranks(
        [ms_per_step, e2e_api_ms, e2e_graph_ms, dec_us, e2e_plain_ms], dev)
    del step_graphs, e2e_graphs, dec_graph, warm_graph, cycle_graph

    # ---- prefill compress (the prefill + batched decode workload): one 4096-token chunk
    # per layer through stief_compress_append (tcgen05 path), timed separately
    compress = None
    if w.name == "prefill_b64" and not args.no_prefill:
        compress = time_prefill_compress(args, len(layers), dev, stream)

    # ---- numbers
    value = job_tokens_per_s(w.B, ws_n, ms_per_step)
    lay0 = layers[0]
    row_bytes = row_bytes_fn(w, args.int8, args.joint, _int4(args))
    bytes_per_dec = int(row_bytes(lay0.rK, lay0.rV) * w.B * w.Hkv * L_dec_mean)
    achieved = bytes_per_dec / (dec_us / 1e6) / 1e9
    peak, peak_kind = _hbm_peak()
    step_bytes = sum(row_bytes(lay.rK, lay.rV) * w.B * w.Hkv for lay in layers) * (
        (ctx_first + ctx_last) / 2)
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
        "dtype": ("int4" if _int4(args) else "int8") if args.int8 else "bf16",
        "data": "synthetic",
        "config": config_dict(w, args, ws_n),
        "hbm_gbs_step": round(step_bytes / (ms_per_step / 1e3) / 1e9, 1),
        "roofline": {
            "kernel": f"stief_decode_kernel ({step_call(args)})",
            "bound": "hbm",
            "achieved": round(achieved, 1),
            "peak": peak,
            "peak_kind": f"{peak_kind} hbm_gbs (copy bandwidth, burst)",
            "unit": "GB/s",
            "frac": round(achieved / peak, 4),
            "traffic": (None if (args.latent or args.unfused or args.paged or args.joint)
                        else _traffic_per_launch(w.name + (("/int4" if _int4(args) else "/int8")
                                                           if args.int8 else ""))),
            "algorithmic_bytes": bytes_per_dec,
            "decode_us": round(dec_us, 3),
            "decode_timing": f"{dec_reps} replays of a graph of {n_dec} back-to-back decode "
                             f"launches over {R} replica(s), context {L_dec}",
            "decode_us_single_launch": round(dec_us_iso, 3),
            "frac_single_launch": round(bytes_per_dec / (dec_us_iso / 1e6) / 1e9 / peak, 4),
        },
        "e2e": {"value": round(job_tokens_per_s(w.B, ws_n, e2e_api_ms), 2), "unit": "tokens/s",
                "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
                "ms_per_step": round(e2e_api_ms, 6),
                "how": "value: every step calls the public API from Python through prepared "
                       "calls (stief.prepare: the binding's argument checks once per buffer "
                       "set, then ctypes into the C entry points, which validate and plan on "
                       "every call) between one H2D copy of the step's inputs from pinned "
                       "memory and one D2H copy of its outputs into pinned memory, CUDA events "
                       "around the K steps; unprepared_value: the same loop with the plain "
                       "binding calls (checks on every call); graph_value: the step captured "
                       "once in a CUDA graph, one replay per step",
                "unprepared_value": round(job_tokens_per_s(w.B, ws_n, e2e_plain_ms), 2),
                "graph_value": round(job_tokens_per_s(w.B, ws_n, e2e_graph_ms), 2),
                "graph_ms_per_step": round(e2e_graph_ms, 6)},
        "gpu_launches": (3 if args.unfused and not args.latent else 1) * len(layers) * K,
        "clocks": clocks,
        "wall_s_timed_region": round(t_wall, 3),
    }
    if compress is not None:
        result["compress"] = compress
    extra = [n for n in args.extra.split(",") if n] if args.extra != "auto" else (
        ["llama31_8b_128k", "llama3_8b_32layer_b16"]
        if w.name == DEFAULT_WORKLOAD and step_call(args) == "stief_append_decode" else [])
    if extra and ws_n == 1:
        result["rooflines"] = [workload_roofline(args, n, dev) for n in extra]
    if (rank == 0 and ws_n == 1 and not args.no_cpu_baseline
            and not (args.latent or args.int8 or args.paged or args.joint)):
        result["cpu_baseline"] = cpu_baseline(w, args.cpu_seconds)
    if ws_n > 1:
        torch.distributed.destroy_process_group()
    if rank == 0:
        print(json.dumps(result), flush=True)


def workload_roofline(args, name: str, dev) -> dict:
    """The fused step's roofline on another workload, measured in the same run: its decode
    kernel (stief_append_decode on layer 0, launches back to back over rotating replicas, like
    the headline's) and its whole step (every layer), each from CUDA-graph replays."""
    import decode_attention_stief_b200 as stief
    w = si.WORKLOADS[name]
    R = replica_count(w)
    n_dec = max(8, R) // R * R
    dec_reps, step_reps = 4, max(3, 12 // R) * R
    grow = 2 * (args.warmup + dec_reps * n_dec // R + step_reps // R) + 64
    reps = [build_state(w, grow, w.seed + 104729 * r, dev) for r in range(R)]
    L_max = reps[0][1]
    reps = [lays for lays, _ in reps]
    g = torch.Generator(device=dev)
    g.manual_seed(w.seed + 1)
    q = torch.randn((w.B, w.Hq, w.d), generator=g, device=dev).to(torch.bfloat16)
    kn = torch.randn((w.B, w.Hkv, 1, w.d), generator=g, device=dev).to(torch.bfloat16)
    vn = torch.randn((w.B, w.Hkv, 1, w.d), generator=g, device=dev).to(torch.bfloat16)
    out = torch.empty((w.B, w.Hq, w.d), dtype=torch.bfloat16, device=dev)
    status = torch.zeros(1, dtype=torch.int32, device=dev)

    def launch(lay):
        stief.stief_append_decode(q, kn, vn, lay.P_K, lay.P_V, lay.k_lat, lay.v_lat, lay.seq_lens,
                                  out, lay.ws, max_seq_len=L_max, dev_status=status)

    def reset():
        for lays in reps:
            for lay in lays:
                lay.seq_lens.fill_(w.L - 1)

    reset()
    for i in range(args.warmup):
        for lay in reps[i % R]:
            launch(lay)
    torch.cuda.synchronize()
    cap = torch.cuda.Stream(device=dev)
    cap.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(cap):
        dec_graph, cycle = torch.cuda.CUDAGraph(), torch.cuda.CUDAGraph()
        with torch.cuda.graph(dec_graph, stream=cap):
            for i in range(n_dec):
                launch(reps[i % R][0])
        with torch.cuda.graph(cycle, stream=cap):
            for r in range(R):
                for lay in reps[r]:
                    launch(lay)
    torch.cuda.synchronize()
    stream = torch.cuda.current_stream()

    def timed(graph, n):
        reset()
        torch.cuda.synchronize()
        _backlog()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for _ in range(n):
            graph.replay()
        e1.record(stream)
        torch.cuda.synchronize()
        return e0.elapsed_time(e1) * 1e3 / n  # us per replay

    dec_us = timed(dec_graph, dec_reps) / n_dec
    step_us = timed(cycle, step_reps // R) / R
    st = stief.stief_read_device_status(status)
    if st != 0:
        raise RuntimeError(f"device status {st:#x} in the {name} roofline")
    del dec_graph, cycle
    rK, rV = w.layer_ranks()[0]
    nbytes = int(2 * (rK + rV) * w.B * w.Hkv * (w.L + dec_reps * n_dec // R / 2))
    peak, kind = _hbm_peak()
    achieved = nbytes / (dec_us / 1e6) / 1e9
    return {"workload": name, "B": w.B, "context": w.L, "layers": len(w.layer_ranks()),
            "ranks_layer0": [rK, rV],
            "decode_us": round(dec_us, 3), "algorithmic_bytes": nbytes,
            "achieved": round(achieved, 1), "peak": peak, "unit": "GB/s",
            "frac": round(achieved / peak, 4), "traffic": _traffic_per_launch(name),
            "step_ms": round(step_us / 1e3, 6),
            "tokens_per_s": round(w.B / (step_us / 1e6), 2),
            "how": f"stief_append_decode on layer 0, {dec_reps} replays of {n_dec} launches back "
                   f"to back over {R} replica(s); step = every layer, {step_reps} steps"}


def time_prefill_compress(args, n_layers: int, dev, stream):
    """Time stief_compress_append of one prefill chunk (B=1, Hkv=8, T=4096, ranks 64/64)
    for every layer, then stief_compress_append_joint_v of the same chunks.  Each layer has
    its own chunk and cache (the chunks of all layers, 537 MB, exceed L2, so every layer's
    chunk streams from HBM without a flush).  Returns a summary dict."""
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

    def timed(fn):
        """Median device time (ms) of one graph replay of fn over every layer."""
        for _ in range(args.warmup):
            lens.zero_()
            fn()
        # the calls of all layers captured in one CUDA graph: the timing is the device's, not
        # the host's launch rate
        torch.cuda.synchronize()
        cap = torch.cuda.Stream(device=dev)
        cap.wait_stream(torch.cuda.current_stream())
        with torch.cuda.stream(cap):
            graph = torch.cuda.CUDAGraph()
            with torch.cuda.graph(graph, stream=cap):
                fn()
        torch.cuda.synchronize()
        reps = max(3, min(args.steps, 20))
        evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
               for _ in range(reps)]
        for r in range(reps):
            lens.zero_()  # every replay appends each layer's chunk to an empty cache
            _backlog()
            evs[r][0].record(stream)
            graph.replay()
            evs[r][1].record(stream)
        torch.cuda.synchronize()
        del graph
        ms = sorted(a.elapsed_time(b) for a, b in evs)
        return ms[len(ms) // 2]

    peak, kind = _hbm_peak()

    def summary(ms_med, bytes_moved, flops):
        return {"us_total": round(ms_med * 1e3, 2), "us_per_layer": round(ms_med * 1e3 / n_layers, 3),
                "algorithmic_bytes": bytes_moved,
                "GBs": round(bytes_moved / (ms_med / 1e3) / 1e9, 1),
                "frac_of_hbm_peak": round(bytes_moved / (ms_med / 1e3) / 1e9 / peak, 4),
                "TFLOPs": round(flops / (ms_med / 1e3) / 1e12, 2),
                "kernel_launches_per_layer": 2}

    ms_med = timed(chunk)
    bytes_moved = n_layers * B * Hkv * T * (2 * d * 2 + 2 * (rK + rV))
    flops = n_layers * B * Hkv * T * 2 * d * (rK + rV)
    out = {"what": f"stief_compress_append of a {T}-token chunk, {Hkv} KV heads, ranks {rK}/{rV}, "
                   f"x{n_layers} layers (tcgen05 path), per-layer chunks (537 MB in all) stream from HBM; "
                   f"the calls of all layers replayed from one CUDA graph"}
    out.update(summary(ms_med, bytes_moved, flops))

    # the same chunks into joint value latents (keys per head, one value row per token over
    # the concatenated heads: a K = Hkv*d contraction), through stief_compress_append_joint_v
    P_VJ = si.to_bf16(si.bases(c["seed"] + 7, 1, Hkv * d, rV)[0]).to(dev)
    vj = [torch.empty((B, T, rV), dtype=torch.bfloat16, device=dev) for _ in range(n_layers)]

    def chunk_joint():
        for li in range(n_layers):
            stief.stief_compress_append_joint_v(ks[li], vs[li], P_K, P_VJ, kl[li], vj[li], lens[li])

    ms_joint = timed(chunk_joint)
    bytes_joint = n_layers * B * T * (Hkv * (2 * d * 2 + 2 * rK) + 2 * rV)
    out["joint"] = {"what": f"stief_compress_append_joint_v of the same chunks (joint value basis "
                            f"[{Hkv * d}][{rV}], tcgen05 path)"}
    out["joint"].update(summary(ms_joint, bytes_joint, flops))
    del vj
    return out


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


def _cpu_model() -> str:
    """The host CPU's model name (first "model name" line of /proc/cpuinfo)."""
    try:
        with open("/proc/cpuinfo") as fh:
            for line in fh:
                if line.startswith("model name"):
                    return line.split(":", 1)[1].strip()
    except OSError:
        pass
    import platform
    return platform.processor() or "unknown"


def cpu_baseline(w: si.Workload, budget_s: float = 20.0):
    """The fp64 oracle (as it stands) on host cores, on a bounded sample of one step:
    layer 0, all sequences and heads, append 1 token + decode, at a context shortened
    so one step takes about budget_s / 2; tokens/s scaled to the full context and layers."""
    import oracle
    threads = min(oracle.max_threads(), w.B * w.Hkv)
    L_s = _sample_context(w, budget_s / 2)
    t = _time_oracle(w, L_s, 0, 2)
    return {"value": round(_oracle_tokens_per_s(w, L_s, t), 4), "unit": "tokens/s",
            "cores": threads, "kind": "oracle", "cpu_model": _cpu_model(),
            "sample": f"layer 0, all {w.B} sequences x {w.Hq} heads, append 1 + decode at "
                      f"context {L_s} (of {w.L}), 2 steps of {t:.2f} s; scaled "
                      f"x{w.L / L_s:.2f} to the context and x{len(w.layer_ranks())} layers"}


def run_profile_launches(args, w: si.Workload):
    """Diagnostics for profilers: N launches of the step's attention kernel (layer 0 of the
    workload, lengths reset before each so every launch sees the same context), then exit."""
    import decode_attention_stief_b200 as stief
    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    layers, L_max = build_state(w, 16, w.seed, dev)
    lay = layers[0]
    g = torch.Generator(device=dev)
    g.manual_seed(w.seed + 1)
    q = torch.randn((w.B, w.Hq, w.d), generator=g, device=dev).to(torch.bfloat16)
    kn = torch.randn((w.B, w.Hkv, w.d), generator=g, device=dev).to(torch.bfloat16)
    vn = torch.randn((w.B, w.Hkv, w.d), generator=g, device=dev).to(torch.bfloat16)
    out = torch.empty_like(q)
    status = torch.zeros(1, dtype=torch.int32, device=dev)
    q_lat = torch.randn((w.B, w.Hq, lay.rK), generator=g, device=dev).to(torch.bfloat16)
    o_lat = torch.empty((w.B, w.Hq, lay.rV), dtype=torch.bfloat16, device=dev)
    if args.int8:  # int8 (4-bit) codes and row scales of layer 0 (synthetic), L_max % 64 == 0
        L8 = (L_max + 63) // 64 * 64
        if _int4(args):
            kq = torch.randint(0, 256, (w.B, w.Hkv, L8, lay.rK // 2), generator=g, device=dev, dtype=torch.uint8)
            vq = torch.randint(0, 256, (w.B, w.Hkv, L8, lay.rV // 2), generator=g, device=dev, dtype=torch.uint8)
        else:
            kq = torch.randint(-127, 128, (w.B, w.Hkv, L8, lay.rK), generator=g, device=dev, dtype=torch.int8)
            vq = torch.randint(-127, 128, (w.B, w.Hkv, L8, lay.rV), generator=g, device=dev, dtype=torch.int8)
        ks = torch.rand((w.B, w.Hkv, L8), generator=g, device=dev) * 0.02
        vs = torch.rand((w.B, w.Hkv, L8), generator=g, device=dev) * 0.02
    if args.joint:  # one joint value basis and one value latent per token (synthetic values)
        js = si.sub_seed(w.seed, 14, 0, 0)
        P_VJ = si.to_bf16(si.bases(js, 1, w.Hkv * w.d, lay.rV)[0]).to(dev)
        v_joint = si.latent_cache_torch(js, w.B, 1, L_max, lay.rV, 1, dev)[:, 0].contiguous()
    for _ in range(args.profile_launches):
        lay.seq_lens.fill_(w.L - 1)
        if args.joint:
            lay.seq_lens.fill_(w.L)
            stief.stief_decode_attention_joint_v(q, lay.P_K, P_VJ, lay.k_lat, v_joint, lay.seq_lens,
                                                 out, lay.ws, max_seq_len=L_max,
                                                 num_splits=args.splits, dev_status=status)
        elif args.int8:
            lay.seq_lens.fill_(w.L)
            (stief.stief_decode_attention_q4 if _int4(args) else stief.stief_decode_attention_q8)(q, lay.P_K, lay.P_V, kq, vq, ks, vs, lay.seq_lens, out,
                                            lay.ws, max_seq_len=L_max, num_splits=args.splits,
                                            dev_status=status)
        elif args.latent:
            lay.seq_lens.fill_(w.L)
            stief.stief_decode_latent(q_lat, lay.k_lat, lay.v_lat, lay.seq_lens, o_lat, lay.ws,
                                      max_seq_len=L_max, num_splits=args.splits,
                                      dev_status=status)
        elif args.unfused:
            lay.seq_lens.fill_(w.L)
            stief.stief_decode_attention(q, lay.P_K, lay.P_V, lay.k_lat, lay.v_lat, lay.seq_lens,
                                         out, lay.ws, max_seq_len=L_max, num_splits=args.splits,
                                         dev_status=status)
        else:
            stief.stief_append_decode(q, kn, vn, lay.P_K, lay.P_V, lay.k_lat, lay.v_lat,
                                      lay.seq_lens, out, lay.ws, max_seq_len=L_max,
                                      num_splits=args.splits, dev_status=status)
    torch.cuda.synchronize()
    st = stief.stief_read_device_status(status)
    if st != 0:
        raise RuntimeError(f"device status {st:#x}")
    print(f"{args.profile_launches} launches of the attention kernel, workload {w.name}, "
          f"context {w.L}", flush=True)


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
        "config": config_dict(w, args, ws_n),
        "cpu_baseline": {"kind": "oracle", "cores": threads, "cpu_model": _cpu_model(),
                         "value": round(value, 4),
                         "unit": "tokens/s", "sample": sample},
        "e2e": {"value": round(value, 4), "unit": "tokens/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }
    print(json.dumps(res), flush=True)


def _free_port() -> int:
    import socket
    with socket.socket(socket.AF_INET, socket.SOCK_STREAM) as sk:
        sk.bind(("127.0.0.1", 0))
        return sk.getsockname()[1]


def launch_ranks(n: int, argv) -> int:
    """Run this script as n ranks of one node (torch.distributed.run on 127.0.0.1); returns the
    launcher's exit code."""
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", f"--nproc-per-node={n}",
           "--master-addr", "127.0.0.1", f"--master-port={_free_port()}",
           os.path.abspath(__file__), *argv]
    return subprocess.call(cmd)


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
    ap.add_argument("--int4", action="store_true",
                    help="time stief_decode_attention_q4 over a 4-bit latent cache (no append; "
                         "ranks multiples of 32)")
    ap.add_argument("--int8", action="store_true",
                    help="time stief_decode_attention_q8 over an int8 latent cache (no append)")
    ap.add_argument("--latent", action="store_true",
                    help="time stief_decode_latent (bases folded into the attention weights) "
                         "instead of the fused append + decode step")
    ap.add_argument("--joint", action="store_true",
                    help="time stief_decode_attention_joint_v: per-head keys, one value latent "
                         "per token shared by the KV heads (no append)")
    ap.add_argument("--paged", action="store_true",
                    help="time stief_append_decode_paged: the fused step over page pools "
                         f"({PAGE_SIZE}-token pages, shuffled block tables)")
    ap.add_argument("--unfused", action="store_true",
                    help="time the step as the two separate calls (append kernel, length "
                         "update, decode) instead of stief_append_decode")
    ap.add_argument("--profile-launches", type=int, default=0,
                    help="diagnostics for profilers: make N launches of the step's attention "
                         "kernel on layer 0 and exit (no timing, no JSON line)")
    ap.add_argument("--clock-window", type=float, default=0.6,
                    help="seconds of untimed decode load before the timed region")
    ap.add_argument("--extra", default="auto",
                    help="comma-separated workloads whose fused-step roofline is measured after "
                         "the headline (auto: the 128k and 32-layer batch-16 workloads beside "
                         "the default 32k one; empty: none)")
    args = ap.parse_args()
    env_world = os.environ.get("WORLD_SIZE")
    if env_world is None and args.gpus > 1:
        # one process per GPU: start the ranks ourselves, as the driver's torchrun would
        sys.exit(launch_ranks(args.gpus, sys.argv[1:]))
    if env_world is not None and int(env_world) != args.gpus:
        ap.error(f"--gpus {args.gpus} but WORLD_SIZE={env_world}: run N ranks with --gpus N")
    if args.warmup < 3:
        ap.error("--warmup must be at least 3")
    modes = [m for m in ("int8", "int4", "latent", "paged", "joint", "unfused") if getattr(args, m)]
    if len(modes) > 1 and modes != ["latent", "joint"]:
        ap.error("--int8, --int4, --latent, --paged, --joint and --unfused are separate modes "
                 "(--latent --joint together time the latent joint-value decode)")
    if args.paged and args.profile_launches > 0:
        ap.error("--profile-launches has no paged mode")
    w = si.WORKLOADS[args.workload]
    if args.int4:
        if any(rK % 32 or rV % 32 for rK, rV in w.layer_ranks()):
            ap.error(f"--int4 needs ranks that are multiples of 32; {w.name} has {w.layer_ranks()}")
        args.int8 = True  # the 4-bit form runs the int8 mode's step with 4-bit codes
    if args.layers > 0:
        import dataclasses
        w = dataclasses.replace(w, layers=min(args.layers, w.layers),
                                ranks=w.ranks[:args.layers] if w.ranks else None)
    if args.profile_launches > 0:
        run_profile_launches(args, w)
    elif args.impl == "reference":
        run_reference(args, w)
    else:
        run_gpu(args, w)


if __name__ == "__main__":
    main()
