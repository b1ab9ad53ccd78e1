"""Joint value latents: stief_decode_attention_joint_v and stief_decode_latent_joint_v (CUDA,
through the C ABI) against the fp64 oracle's decode_joint_v and decode_latent_joint_v.

The values of a token's KV heads are factored together (STAR-KV technical summary,
"Metodologia" item 2): one latent row per token, v_joint [B][L_max][rV], shared by every KV
head; KV head g rebuilds its values from rows [g*d, (g+1)*d) of P_VJ [Hkv*d][rV].  Keys keep
one basis per KV head.  Tolerance as for the per-head decode: 2e-2 * ||o||_inf.
"""
import numpy as np
import pytest
import torch

import decode_attention_stief_b200 as stief
import oracle
import stief_inputs as si
from gpu_util import assert_decode_close, f64, gpu_decode

pytestmark = pytest.mark.gpu
DEV = torch.device("cuda")


def _case(B, Hq, Hkv, rK, rV, L_max, seed, d=128):
    q = si.queries(seed, B, Hq, d)
    P_K = si.to_bf16(si.bases(seed, Hkv, d, rK))
    P_VJ = si.to_bf16(si.bases(seed + 1, 1, Hkv * d, rV)[0])
    k = si.latent_cache(seed, B, Hkv, L_max, rK, 0)
    v = si.latent_cache(seed, B, 1, L_max, rV, 1)[:, 0].contiguous()
    return q, P_K, P_VJ, k, v


def _ws(B, Hq, Hkv, rV, max_seq_len):
    return stief.workspace_for(B, Hq, Hkv, rV, max_seq_len)


def _gpu_joint(q, P_K, P_VJ, k, v, lens, num_splits=0, max_seq_len=None, expect_status=0):
    q, P_K, P_VJ, k, v = (x.to(DEV).contiguous() for x in (q, P_K, P_VJ, k, v))
    B, Hq, d = q.shape
    Hkv, rV = P_K.shape[0], P_VJ.shape[1]
    if max_seq_len is None:
        max_seq_len = int(max(lens)) if len(lens) else 0
    out = torch.full((B, Hq, d), float("nan"), dtype=torch.bfloat16, device=DEV)
    status = torch.zeros(1, dtype=torch.int32, device=DEV)
    stief.stief_decode_attention_joint_v(q, P_K, P_VJ, k, v,
                                         torch.as_tensor(np.asarray(lens, np.int32)).to(DEV),
                                         out, _ws(B, Hq, Hkv, rV, max_seq_len), max_seq_len,
                                         num_splits=num_splits, dev_status=status)
    assert stief.stief_read_device_status(status) == expect_status
    return out.cpu()


def _gpu_latent_joint(q_lat, k, v, lens, num_splits=0, max_seq_len=None):
    q_lat, k, v = (x.to(DEV).contiguous() for x in (q_lat, k, v))
    B, Hq, rK = q_lat.shape
    Hkv, rV = k.shape[1], v.shape[2]
    if max_seq_len is None:
        max_seq_len = int(max(lens)) if len(lens) else 0
    out = torch.full((B, Hq, rV), float("nan"), dtype=torch.bfloat16, device=DEV)
    status = torch.zeros(1, dtype=torch.int32, device=DEV)
    stief.stief_decode_latent_joint_v(q_lat, k, v,
                                      torch.as_tensor(np.asarray(lens, np.int32)).to(DEV), out,
                                      _ws(B, Hq, Hkv, rV, max_seq_len), max_seq_len,
                                      num_splits=num_splits, dev_status=status)
    assert stief.stief_read_device_status(status) == 0
    return out.cpu()


def _oracle(q, P_K, P_VJ, k, v, lens):
    return oracle.decode_joint_v(f64(q), f64(P_K), f64(P_VJ), f64(k), f64(v),
                                 np.asarray(lens, np.int32))


@pytest.mark.parametrize("num_splits", [0, 1, 3, 7])
def test_ragged_batch_splits(num_splits):
    lens = [900, 33, 0, 257, 1]
    q, P_K, P_VJ, k, v = _case(5, 16, 4, 64, 64, 900, 7100)
    got = _gpu_joint(q, P_K, P_VJ, k, v, lens, num_splits=num_splits)
    assert_decode_close(got, _oracle(q, P_K, P_VJ, k, v, lens))
    assert torch.all(got[2].float() == 0), "empty sequence must give exactly zero"


@pytest.mark.parametrize("L", [1, 31, 32, 33, 64, 65, 1000])
def test_tile_boundaries(L):
    q, P_K, P_VJ, k, v = _case(2, 8, 2, 32, 48, L, 7200 + L)  # ranks 32/48: 64-token tiles
    got = _gpu_joint(q, P_K, P_VJ, k, v, [L, max(1, L // 2)])
    assert_decode_close(got, _oracle(q, P_K, P_VJ, k, v, [L, max(1, L // 2)]))


@pytest.mark.parametrize("rK,rV", [(16, 16), (16, 128), (128, 16), (48, 96), (128, 128)])
def test_all_ranks(rK, rV):
    q, P_K, P_VJ, k, v = _case(2, 8, 2, rK, rV, 300, 7300 + rK + rV)
    got = _gpu_joint(q, P_K, P_VJ, k, v, [300, 129])
    assert_decode_close(got, _oracle(q, P_K, P_VJ, k, v, [300, 129]))


@pytest.mark.parametrize("Hq,Hkv", [(8, 8), (32, 8), (48, 1), (6, 2)])
def test_gqa_groups(Hq, Hkv):
    q, P_K, P_VJ, k, v = _case(3, Hq, Hkv, 64, 48, 200, 7400 + Hq + Hkv)
    got = _gpu_joint(q, P_K, P_VJ, k, v, [200, 77, 150])
    assert_decode_close(got, _oracle(q, P_K, P_VJ, k, v, [200, 77, 150]))


@pytest.mark.parametrize("num_splits", [0, 1, 4])
def test_latent_joint_matches_oracle(num_splits):
    B, Hq, Hkv, rK, rV, L = 3, 32, 8, 64, 96, 700
    q_lat = si.queries(7500, B, Hq, rK)
    k = si.latent_cache(7500, B, Hkv, L, rK, 0)
    v = si.latent_cache(7500, B, 1, L, rV, 1)[:, 0].contiguous()
    lens = [700, 64, 0]
    got = _gpu_latent_joint(q_lat, k, v, lens, num_splits=num_splits)
    want = oracle.decode_latent_joint_v(f64(q_lat), f64(k), f64(v), np.asarray(lens, np.int32))
    assert_decode_close(got, want)
    assert torch.all(got[2].float() == 0)


def test_block_diagonal_basis_equals_the_per_head_decode():
    """P_VJ = blockdiag(P_V[0], P_V[1]) with the per-head latents side by side: the joint call
    and the per-head call attend over the same values (both on the GPU, and the oracle)."""
    B, Hq, Hkv, rK, r, L = 2, 8, 2, 64, 64, 400
    q = si.queries(7600, B, Hq, 128)
    P_K, P_V = si.bases_bf16(7600, Hkv, 128, rK, r)
    k = si.latent_cache(7600, B, Hkv, L, rK, 0)
    v = si.latent_cache(7600, B, Hkv, L, r, 1)
    P_VJ = torch.zeros((Hkv * 128, Hkv * r), dtype=torch.bfloat16)
    for g in range(Hkv):
        P_VJ[g * 128:(g + 1) * 128, g * r:(g + 1) * r] = P_V[g]
    v_joint = torch.cat([v[:, g] for g in range(Hkv)], dim=-1).contiguous()  # [B][L][Hkv*r]
    lens = [400, 123]
    got = _gpu_joint(q, P_K, P_VJ, k, v_joint, lens)
    per_head = gpu_decode(q, P_K, P_V, k, v, lens)
    want = oracle.decode(f64(q), f64(P_K), f64(P_V), f64(k), f64(v), np.asarray(lens, np.int32))
    assert_decode_close(got, want)
    assert_decode_close(per_head, want)


def test_multi_wave_grid():
    """40 x 8 units: the joint decode in the two-CTAs-per-SM plan."""
    B, Hq, Hkv, rK, rV, L = 40, 32, 8, 64, 64, 320
    rng = np.random.default_rng(7700)
    lens = rng.integers(1, L, size=B).tolist()
    lens[5] = 0
    q, P_K, P_VJ, k, v = _case(B, Hq, Hkv, rK, rV, L, 7700)
    got = _gpu_joint(q, P_K, P_VJ, k, v, lens, max_seq_len=L)
    assert_decode_close(got, _oracle(q, P_K, P_VJ, k, v, lens))
    assert torch.all(got[5].float() == 0)


def test_shape_errors_are_refused_before_launch():
    q, P_K, P_VJ, k, v = _case(1, 8, 2, 32, 32, 64, 7800)
    with pytest.raises(ValueError):   # a per-head value cache where the joint one is expected
        _gpu_joint(q, P_K, P_VJ, k, k, [64])
