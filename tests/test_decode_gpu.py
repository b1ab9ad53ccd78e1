"""Decode parity: stief_decode_attention (CUDA, through the C ABI) against the fp64 oracle.

Tolerance (the benchmark spec): max |o_gpu - o_oracle| <= 2e-2 * ||o_oracle||_inf for bf16
storage with fp32 accumulation.  Sizes span several warp tiles, several splits
and ragged tails; edge cases cover empty sequences, single tokens, poisoned
slots beyond the length, every supported rank and several GQA group sizes.
"""
import numpy as np
import pytest
import torch

import stief_inputs as si
from gpu_util import (assert_decode_close, decode_error, gpu_decode, make_decode_case,
                      oracle_decode)

pytestmark = pytest.mark.gpu


def _run(B, Hq, Hkv, rK, rV, L_max, lens, seed, num_splits=0, q_scale=1.0):
    case = make_decode_case(B, Hq, Hkv, rK, rV, L_max, seed, q_scale=q_scale)
    got = gpu_decode(*case, lens, num_splits=num_splits)
    want = oracle_decode(*case, lens)
    return got, want, case


def test_tiny_config():
    w = si.WORKLOADS["tiny"]
    got, want, _ = _run(w.B, w.Hq, w.Hkv, w.rK, w.rV, w.L, [w.L], w.seed)
    assert_decode_close(got, want)


@pytest.mark.parametrize("num_splits", [0, 1, 3, 6])
def test_ragged_batch_multi_tile(num_splits):
    lens = [700, 33, 0, 257]
    got, want, _ = _run(4, 8, 2, 32, 48, 700, lens, 7, num_splits=num_splits)
    assert_decode_close(got, want)
    assert torch.all(got[2].float() == 0), "empty sequence must give exactly zero"


@pytest.mark.parametrize("L", [1, 2, 31, 32, 33, 63, 64, 65, 255, 256, 257, 1000])
def test_tile_boundaries(L):
    got, want, _ = _run(1, 4, 1, 64, 64, L, [L], 100 + L)
    assert_decode_close(got, want)


@pytest.mark.parametrize("rK,rV", [(16, 16), (16, 128), (128, 16), (32, 48), (48, 32),
                                   (64, 96), (80, 112), (96, 64), (112, 80), (128, 128)])
def test_all_ranks(rK, rV):
    got, want, _ = _run(2, 8, 2, rK, rV, 300, [300, 129], 200 + rK + rV)
    assert_decode_close(got, want)


@pytest.mark.parametrize("Hq,Hkv", [(8, 8), (16, 8), (24, 8), (32, 8), (64, 8), (32, 2),
                                    (48, 1), (6, 2)])
def test_gqa_groups(Hq, Hkv):
    got, want, _ = _run(2, Hq, Hkv, 64, 64, 200, [200, 77], 300 + Hq + Hkv)
    assert_decode_close(got, want)


@pytest.mark.parametrize("q_scale", [8.0, 30.0])
def test_peaked_attention(q_scale):
    got, want, _ = _run(2, 8, 2, 64, 64, 500, [500, 300], 400, q_scale=q_scale)
    assert_decode_close(got, want)


def test_needle_tokens():
    """Keys built to align with their query at known positions: a wrong scale, row index or
    head mapping moves weight away from the needles and changes the output."""
    B, Hq, Hkv, d, rK, rV, L = 1, 8, 2, 128, 64, 64, 900
    seed = 500
    q, P_K, P_V, k_lat, v_lat = make_decode_case(B, Hq, Hkv, rK, rV, L, seed)
    # full-dimension needle keys: k = 6 * q_h / |q_h| projected by each side
    import oracle
    from gpu_util import f64
    pk = f64(P_K)
    kl = f64(k_lat)
    rng = np.random.default_rng(1)
    for h in range(Hq):
        g = h // (Hq // Hkv)
        t = int(rng.integers(0, L))
        qh = f64(q)[0, h]
        kl[0, g, t] = oracle.project((6.0 * np.sqrt(d) * qh / np.linalg.norm(qh))[None], pk[g])[0]
    k_lat = si.to_bf16(kl)
    lens = [L]
    got = gpu_decode(q, P_K, P_V, k_lat, v_lat, lens)
    want = oracle_decode(q, P_K, P_V, k_lat, v_lat, lens)
    assert_decode_close(got, want)


def test_poisoned_slots_beyond_length_are_never_read():
    B, Hq, Hkv, rK, rV, L_max = 2, 8, 2, 32, 64, 400
    lens = [250, 37]
    q, P_K, P_V, k_lat, v_lat = make_decode_case(B, Hq, Hkv, rK, rV, L_max, 600)
    clean = gpu_decode(q, P_K, P_V, k_lat, v_lat, lens)
    for b, L in enumerate(lens):
        k_lat[b, :, L:] = float("nan")
        v_lat[b, :, L:] = float("inf")
    dirty = gpu_decode(q, P_K, P_V, k_lat, v_lat, lens)
    assert torch.equal(clean, dirty)
    assert torch.all(torch.isfinite(dirty.float()))


def test_deterministic_bits():
    case = make_decode_case(2, 32, 8, 64, 64, 3000, 700)
    a = gpu_decode(*case, [3000, 1500])
    b = gpu_decode(*case, [3000, 1500])
    assert torch.equal(a, b)


def test_split_count_invariance():
    case = make_decode_case(1, 32, 8, 64, 64, 4096, 800)
    outs = [gpu_decode(*case, [4096], num_splits=s) for s in (1, 2, 5, 18, 32)]
    want = oracle_decode(*case, [4096])
    for o in outs:
        assert_decode_close(o, want)
    ref = outs[0].double()
    for o in outs[1:]:
        assert float((o.double() - ref).abs().max()) <= 2e-2 * float(ref.abs().max())


def test_bad_length_is_reported_and_gives_zero():
    case = make_decode_case(2, 8, 2, 32, 32, 64, 900)
    # second sequence claims more rows than the cache holds: output zero, status bit set
    import decode_attention_stief_b200 as stief
    got = gpu_decode(*case, [64, 65], max_seq_len=64, expect_status=stief.DEV_BAD_LENGTH)
    want = oracle_decode(*case, [64, 0])
    assert_decode_close(got, want)
    assert torch.all(got[1].float() == 0)


def test_status_word_stays_clear_on_success():
    case = make_decode_case(1, 4, 1, 64, 64, 128, 901)
    gpu_decode(*case, [128], expect_status=0)


def test_workspace_counters_return_to_zero_and_partials_may_hold_garbage():
    """The ticket counters are the only workspace state that must be zero on entry; every
    completed call leaves them at zero, whatever the partial-state area holds."""
    import decode_attention_stief_b200 as stief
    case = make_decode_case(2, 32, 8, 64, 48, 4096, 950)
    dev = torch.device("cuda")
    q, P_K, P_V, k_lat, v_lat = (x.to(dev) for x in case)
    lens = torch.tensor([4096, 2500], dtype=torch.int32, device=dev)
    ws = stief.workspace_for(2, 32, 8, 48, 4096)
    counter_bytes = 256  # 16 units x 4 bytes, padded to 256
    ws[counter_bytes:].fill_(0xFF)
    want = oracle_decode(*case, [4096, 2500])
    for splits in (9, 9, 32, 1, 5):
        out = torch.empty((2, 32, 128), dtype=torch.bfloat16, device=dev)
        stief.stief_decode_attention(q, P_K, P_V, k_lat, v_lat, lens, out, ws, 4096,
                                     num_splits=splits)
        torch.cuda.synchronize()
        assert int(ws[:counter_bytes].count_nonzero()) == 0
        assert_decode_close(out.cpu(), want)


@pytest.mark.parametrize("rK,rV", [(64, 64), (32, 96), (32, 48)])
def test_multi_wave_grid_two_ctas_per_sm(rK, rV):
    """More (sequence, KV head) units than SMs with one split: the planner runs two CTAs per
    SM with a smaller ring; ragged lengths, an empty sequence and tile tails included."""
    B = 40  # 40 x 8 KV heads = 320 units, more than the 148 SMs
    rng = np.random.default_rng(990 + rK)
    lens = rng.integers(1, 300, size=B).tolist()
    lens[3] = 0
    lens[7] = 300
    got, want, _ = _run(B, 32, 8, rK, rV, 300, lens, 991 + rK + rV)
    assert_decode_close(got, want)
    assert torch.all(got[3].float() == 0)
