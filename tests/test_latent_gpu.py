"""Latent decode parity: stief_decode_latent (CUDA, through the C ABI) against the fp64
oracle's decode_latent.

The latent decode is the deployment form with the bases folded into the attention weights
(StiefAttention technical summary, "Mecanismo Central" item 5, last sentence): q~ comes in
[B][Hq][rK], o~ goes out [B][Hq][rV].  Tolerance as for the decode: max |o~_gpu - o~| <=
2e-2 * ||o~||_inf.  The query rows are what a folded query weight produces for N(0, 1)
queries and orthonormal bases: N(0, 1) in r_K dimensions.
"""
import numpy as np
import pytest
import torch

import decode_attention_stief_b200 as stief
import oracle
import stief_inputs as si
from gpu_util import DECODE_TOL, assert_decode_close, decode_error, f64, gpu_decode

pytestmark = pytest.mark.gpu


def _case(B, Hq, Hkv, rK, rV, L_max, seed, q_scale=1.0):
    q = si.queries(seed, B, Hq, rK, scale=q_scale)
    k = si.latent_cache(seed, B, Hkv, L_max, rK, 0)
    v = si.latent_cache(seed, B, Hkv, L_max, rV, 1)
    return q, k, v


def _gpu_latent(q, k, v, lens, num_splits=0, max_seq_len=None, ws=None, expect_status=0):
    dev = torch.device("cuda")
    q, k, v = (x.to(dev).contiguous() for x in (q, k, v))
    B, Hq, rK = q.shape
    Hkv, rV = k.shape[1], v.shape[3]
    if max_seq_len is None:
        max_seq_len = int(max(lens)) if len(lens) else 0
    lens_t = torch.as_tensor(np.asarray(lens, dtype=np.int32)).to(dev)
    out = torch.full((B, Hq, rV), float("nan"), dtype=torch.bfloat16, device=dev)
    if ws is None:
        ws = stief.workspace_for(B, Hq, Hkv, rV, max_seq_len)
    status = torch.zeros(1, dtype=torch.int32, device=dev)
    stief.stief_decode_latent(q, k, v, lens_t, out, ws, max_seq_len, num_splits=num_splits,
                              dev_status=status)
    assert stief.stief_read_device_status(status) == expect_status
    return out.cpu()


def _oracle(q, k, v, lens):
    return oracle.decode_latent(f64(q), f64(k), f64(v), np.asarray(lens, np.int32), d=128)


@pytest.mark.parametrize("num_splits", [0, 1, 3, 7])
def test_ragged_batch_splits(num_splits):
    lens = [900, 33, 0, 257, 1]
    q, k, v = _case(5, 16, 4, 64, 64, 900, 4100)
    got = _gpu_latent(q, k, v, lens, num_splits=num_splits)
    assert_decode_close(got, _oracle(q, k, v, lens))
    assert torch.all(got[2].float() == 0), "empty sequence must give exactly zero"


@pytest.mark.parametrize("L", [1, 2, 31, 32, 33, 64, 65, 257, 1000])
def test_tile_boundaries(L):
    q, k, v = _case(1, 4, 1, 32, 48, L, 4200 + L)  # ranks 32/48: 64-token tiles
    got = _gpu_latent(q, k, v, [L])
    assert_decode_close(got, _oracle(q, k, v, [L]))


@pytest.mark.parametrize("rK,rV", [(16, 16), (16, 128), (128, 16), (32, 48), (48, 32),
                                   (64, 96), (96, 64), (128, 128)])
def test_all_ranks(rK, rV):
    q, k, v = _case(2, 8, 2, rK, rV, 300, 4300 + rK + rV)
    got = _gpu_latent(q, k, v, [300, 129])
    assert_decode_close(got, _oracle(q, k, v, [300, 129]))


@pytest.mark.parametrize("Hq,Hkv", [(8, 8), (32, 8), (64, 8), (48, 1), (6, 2)])
def test_gqa_groups(Hq, Hkv):
    q, k, v = _case(2, Hq, Hkv, 64, 48, 200, 4400 + Hq + Hkv)
    got = _gpu_latent(q, k, v, [200, 77])
    assert_decode_close(got, _oracle(q, k, v, [200, 77]))


@pytest.mark.parametrize("q_scale", [8.0, 30.0])
def test_peaked_softmax_and_needle(q_scale):
    """Large scores and a planted needle: a wrong scale or head mapping shows."""
    q, k, v = _case(2, 8, 2, 64, 64, 500, 4500, q_scale=q_scale)
    k = k.clone()
    for b in range(2):
        for g in range(2):
            k[b, g, 123 + 50 * g] = q[b, 4 * g] / q[b, 4 * g].float().norm() * 8.0
    got = _gpu_latent(q, k, v, [500, 400])
    assert_decode_close(got, _oracle(q, k, v, [500, 400]))


def test_folding_identity_against_the_full_decode():
    """decode_latent(bf16(q P_K)) P_V^T is the full decode up to the bf16 rounding of q~."""
    B, Hq, Hkv, rK, rV, L = 2, 32, 8, 64, 48, 700
    P_K, P_V = si.bases_bf16(4600, Hkv, 128, rK, rV)
    q = si.queries(4601, B, Hq, 128)
    k = si.latent_cache(4602, B, Hkv, L, rK, 0)
    v = si.latent_cache(4602, B, Hkv, L, rV, 1)
    G = Hq // Hkv
    qf, pk, pv = q.double(), P_K.double(), P_V.double()
    q_lat = torch.stack([torch.stack([qf[b, h] @ pk[h // G] for h in range(Hq)])
                         for b in range(B)]).to(torch.bfloat16)
    lens = [L, 400]
    o_lat = _gpu_latent(q_lat, k, v, lens).double()
    up = torch.stack([torch.stack([o_lat[b, h] @ pv[h // G].T for h in range(Hq)])
                      for b in range(B)])
    full = gpu_decode(q, P_K, P_V, k, v, lens)
    want = oracle.decode(f64(q), f64(P_K), f64(P_V), f64(k), f64(v), np.asarray(lens, np.int32))
    assert decode_error(full, want) <= DECODE_TOL
    assert decode_error(up.to(torch.bfloat16), want) <= DECODE_TOL


def test_counters_stay_zero_and_out_of_range_length_is_flagged():
    """The workspace is shared with the decode: its counters return to zero; a length above
    max_seq_len sets STIEF_DEV_BAD_LENGTH and gives zeros for that sequence."""
    q, k, v = _case(2, 8, 2, 64, 64, 600, 4700)
    ws = stief.workspace_for(2, 8, 2, 64, 600)
    for s in (4, 1, 3):
        got = _gpu_latent(q, k, v, [600, 300], num_splits=s, ws=ws)
        assert_decode_close(got, _oracle(q, k, v, [600, 300]))
        assert int(ws[:256].count_nonzero()) == 0
    got = _gpu_latent(q, k, v, [600, 700], max_seq_len=600, ws=stief.workspace_for(2, 8, 2, 64, 600),
                      expect_status=stief.DEV_BAD_LENGTH)
    assert torch.all(got[1].float() == 0)


@pytest.mark.parametrize("name", ["llama3_8b_32k", "llama31_8b_128k"])
def test_full_size_one_layer(name):
    """The benchmark shapes at full context, automatic splits, every head checked exactly."""
    w = si.WORKLOADS[name]
    dev = torch.device("cuda")
    seed = si.sub_seed(w.seed, 47)
    k = si.latent_cache_torch(seed, w.B, w.Hkv, w.L, w.rK, 0, dev)
    v = si.latent_cache_torch(seed, w.B, w.Hkv, w.L, w.rV, 1, dev)
    q = si.queries_torch(seed + 1, w.B, w.Hq, w.rK, dev)
    got = _gpu_latent(q, k, v, [w.L] * w.B)
    want = _oracle(q, k, v, [w.L] * w.B)
    err = decode_error(got, want)
    print(f"\n  {name} latent decode: max|err| / ||o~||_inf = {err:.3e}")
    assert err <= DECODE_TOL


def test_multi_wave_grid_two_ctas_per_sm():
    """The latent decode on a grid of more units than SMs (two CTAs per SM)."""
    lens = [257, 1, 0, 300] * 10
    q, k, v = _case(40, 32, 8, 64, 64, 300, 4800)
    got = _gpu_latent(q, k, v, lens)
    assert_decode_close(got, _oracle(q, k, v, lens))
