"""Parity on the five benchmark configurations at their full sizes, in the launch
configuration the benchmark uses (stief_append_decode, automatic splits): one decode step of
every checked layer against the fp64 oracle run on the same cache (the oracle's own append
of the new rows, then its decode).  Cheap configurations are checked whole; for the 32-layer
ones a sample of layers and sequences is checked exactly (the GPU still runs the full batch).
The measured errors are printed (pytest -s) for the record.
"""
import numpy as np
import pytest
import torch

import decode_attention_stief_b200 as stief
import oracle
import stief_inputs as si
from gpu_util import DECODE_TOL, decode_error, f64

pytestmark = pytest.mark.gpu


def _check_layer(w, li, rK, rV, seqs):
    dev = torch.device("cuda")
    L0 = w.L - 1  # the step appends the L-th token
    L_max = w.L + 64
    seed = si.sub_seed(w.seed, 40, li)
    P_K, P_V = si.bases_bf16(seed, w.Hkv, w.d, rK, rV)
    k_lat = si.latent_cache_torch(seed + 1, w.B, w.Hkv, L_max, rK, 0, dev)
    v_lat = si.latent_cache_torch(seed + 2, w.B, w.Hkv, L_max, rV, 1, dev)
    q = si.queries_torch(seed + 3, w.B, w.Hq, w.d, dev)
    g = torch.Generator(device=dev)
    g.manual_seed(seed + 4)
    kn = torch.randn((w.B, w.Hkv, w.d), generator=g, device=dev).to(torch.bfloat16)
    vn = torch.randn((w.B, w.Hkv, w.d), generator=g, device=dev).to(torch.bfloat16)
    # oracle inputs for the sampled sequences, taken before the step writes row L0
    ok_, ov_ = f64(k_lat[seqs, :, :L0 + 1]), f64(v_lat[seqs, :, :L0 + 1])
    lens = torch.full((w.B,), L0, dtype=torch.int32, device=dev)
    out = torch.empty((w.B, w.Hq, w.d), dtype=torch.bfloat16, device=dev)
    ws = stief.workspace_for(w.B, w.Hq, w.Hkv, rV, L_max)
    status = torch.zeros(1, dtype=torch.int32, device=dev)
    stief.stief_append_decode(q, kn, vn, P_K.to(dev), P_V.to(dev), k_lat, v_lat, lens, out, ws,
                              L_max, dev_status=status)
    assert stief.stief_read_device_status(status) == 0
    assert torch.all(lens == L0 + 1)
    Pk, Pv = f64(P_K), f64(P_V)
    for i, b in enumerate(seqs):  # the oracle's append: row L0 = RNE_bf16(x . P)
        for h in range(w.Hkv):
            ok_[i, h, L0] = oracle.project(f64(kn[b, h])[None], Pk[h], round_to_bf16=True)[0]
            ov_[i, h, L0] = oracle.project(f64(vn[b, h])[None], Pv[h], round_to_bf16=True)[0]
    want = oracle.decode(f64(q[seqs]), Pk, Pv, ok_, ov_, np.full(len(seqs), L0 + 1, np.int32))
    err = decode_error(out[seqs].cpu(), want)
    print(f"\n  {w.name} layer {li} ranks {rK}/{rV}: max|err| / ||o||_inf = {err:.3e} "
          f"({len(seqs)} of {w.B} sequences, all {w.Hq} heads)")
    assert err <= DECODE_TOL
    return err


def test_config1_tiny():
    w = si.WORKLOADS["tiny"]
    _check_layer(w, 0, w.rK, w.rV, list(range(w.B)))


def test_config2_llama3_8b_32k():
    w = si.WORKLOADS["llama3_8b_32k"]
    _check_layer(w, 0, w.rK, w.rV, [0])


def test_config3_32layer_b16_sampled_layers():
    w = si.WORKLOADS["llama3_8b_32layer_b16"]
    ranks = w.layer_ranks()
    for li in (0, 3, 13, 31):  # rank pairs (48,32), (96,48), (32,96), (96,48)
        _check_layer(w, li, *ranks[li], seqs=[0, 15])


def test_config4_llama31_8b_128k():
    w = si.WORKLOADS["llama31_8b_128k"]
    _check_layer(w, 0, w.rK, w.rV, [0])


def test_config5_prefill_b64_decode_sampled():
    w = si.WORKLOADS["prefill_b64"]
    for li in (0, 31):
        _check_layer(w, li, w.rK, w.rV, seqs=[0, 37, 63])
