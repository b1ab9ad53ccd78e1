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


# ----------------------------------------------------------------------------- joint compress

CANARY = 0x7FC1  # a quiet-NaN bf16 pattern: any stray write changes it


def _canary(shape):
    t = torch.full(shape, CANARY, dtype=torch.int16, device=DEV)
    return t.view(torch.bfloat16)


def _compress_joint(k_new, v_new, P_K, P_VJ, L_max, lens):
    B, Hkv, T, d = k_new.shape
    rK, rV = P_K.shape[2], P_VJ.shape[1]
    k_lat = _canary((B, Hkv, L_max, rK))
    v_joint = _canary((B, L_max, rV))
    lens_t = torch.as_tensor(np.asarray(lens, np.int32)).to(DEV)
    status = torch.zeros(1, dtype=torch.int32, device=DEV)
    stief.stief_compress_append_joint_v(k_new.to(DEV), v_new.to(DEV), P_K.to(DEV), P_VJ.to(DEV),
                                        k_lat, v_joint, lens_t, dev_status=status)
    st = stief.stief_read_device_status(status)
    return k_lat.cpu(), v_joint.cpu(), lens_t.cpu().numpy(), st


def _selector_basis(Hkv, d, r):
    """[Hkv*d][r] with column c = the unit vector of head c % Hkv, dimension c // Hkv: every
    stored coordinate is one input coordinate, from heads in turn (exact in bf16)."""
    P = np.zeros((Hkv * d, r))
    for c in range(r):
        P[(c % Hkv) * d + c // Hkv, c] = 1.0
    return si.to_bf16(P)


@pytest.mark.parametrize("T", [1, 5, 8, 20])
def test_compress_selector_bases_bit_exact(T):
    """Selector bases: each stored value is one input coordinate, so the GPU's rows equal the
    oracle's bit for bit (which head each column reads is fixed by the concatenation order)."""
    B, Hkv, d, rK, rV, L_max = 2, 4, 128, 32, 48, 40
    k_new, v_new = si.full_kv(7900 + T, B, Hkv, T, d)
    P_K = torch.stack([_selector_basis(1, d, rK) for _ in range(Hkv)])
    P_VJ = _selector_basis(Hkv, d, rV)
    lens = [0, 11]
    gk, gv, glens, st = _compress_joint(k_new, v_new, P_K, P_VJ, L_max, lens)
    assert st == 0 and glens.tolist() == [L + T for L in lens]
    wk, wv, wl, nbad = oracle.compress_append_joint_v(
        f64(k_new), f64(v_new), f64(P_K), f64(P_VJ), np.zeros((B, Hkv, L_max, rK)),
        np.zeros((B, L_max, rV)), np.asarray(lens, np.int32))
    assert nbad == 0 and wl.tolist() == glens.tolist()
    for b, L in enumerate(lens):
        assert np.array_equal(f64(gk[b, :, L:L + T]), wk[b, :, L:L + T])
        assert np.array_equal(f64(gv[b, L:L + T]), wv[b, L:L + T])
        keep = np.ones(L_max, bool)
        keep[L:L + T] = False
        assert torch.all(gk[b][:, keep].view(torch.int16) == CANARY)
        assert torch.all(gv[b][keep].view(torch.int16) == CANARY)


@pytest.mark.parametrize("T", [3, 130])
def test_compress_general_bases_within_the_fp32_bound(T):
    """General bases: the fp32 sum of Hkv*d products, rounded once to bf16, against the exact
    product: within half a bf16 ulp plus the fp32 accumulation bound K * 2^-23 * sum|x||p|."""
    B, Hkv, d, rK, rV, L_max = 1, 8, 128, 64, 64, 160
    k_new, v_new = si.full_kv(8000 + T, B, Hkv, T, d)
    P_K = si.to_bf16(si.bases(8000, Hkv, d, rK))
    P_VJ = si.to_bf16(si.bases(8001, 1, Hkv * d, rV)[0])
    gk, gv, glens, st = _compress_joint(k_new, v_new, P_K, P_VJ, L_max, [7])
    assert st == 0 and glens.tolist() == [7 + T]
    x = np.ascontiguousarray(np.transpose(f64(v_new[0]), (1, 0, 2)).reshape(T, Hkv * d))
    P = f64(P_VJ)
    exact = x @ P
    bound = 2.0 ** -8 * np.abs(exact) + Hkv * d * 2.0 ** -23 * (np.abs(x) @ np.abs(P)) + 1e-30
    got = f64(gv[0, 7:7 + T])
    assert np.all(np.abs(got - exact) <= bound)
    want = oracle.compress_append_joint_v(f64(k_new), f64(v_new), f64(P_K), f64(P_VJ),
                                          np.zeros((B, Hkv, L_max, rK)), np.zeros((B, L_max, rV)),
                                          np.array([7], np.int32))[1][0, 7:7 + T]
    assert np.mean(got == want) > 0.95
    for h in range(Hkv):
        ek = f64(k_new[0, h]) @ f64(P_K[h])
        kb = 2.0 ** -8 * np.abs(ek) + d * 2.0 ** -23 * (np.abs(f64(k_new[0, h])) @ np.abs(f64(P_K[h])))
        assert np.all(np.abs(f64(gk[0, h, 7:7 + T]) - ek) <= kb + 1e-30)


def test_compress_refuses_full_and_bad_sequences():
    """A sequence whose rows would pass L_max, and one with a negative length, are skipped
    (nothing written, length unchanged) and reported; the others are appended."""
    B, Hkv, d, rK, rV, L_max, T = 3, 2, 128, 32, 32, 16, 4
    k_new, v_new = si.full_kv(8100, B, Hkv, T, d)
    P_K = si.to_bf16(si.bases(8100, Hkv, d, rK))
    P_VJ = si.to_bf16(si.bases(8101, 1, Hkv * d, rV)[0])
    gk, gv, glens, st = _compress_joint(k_new, v_new, P_K, P_VJ, L_max, [13, -1, 12])
    assert st == (stief.DEV_CAPACITY_OVERFLOW | stief.DEV_BAD_LENGTH)
    assert glens.tolist() == [13, -1, 16]
    for b in (0, 1):
        assert torch.all(gk[b].view(torch.int16) == CANARY)
        assert torch.all(gv[b].view(torch.int16) == CANARY)
    assert not torch.any(gv[2, 12:16].view(torch.int16) == CANARY)


def test_compress_then_decode_joint_end_to_end():
    """A prefill chunk and one decode-step token into a joint cache, then the joint decode,
    against the oracle's joint compress and decode."""
    B, Hq, Hkv, d, rK, rV, L_max = 2, 32, 8, 128, 64, 96, 200
    k_pre, v_pre = si.full_kv(8200, B, Hkv, 150, d)
    k_new, v_new = si.full_kv(8201, B, Hkv, 1, d)
    P_K = si.to_bf16(si.bases(8200, Hkv, d, rK))
    P_VJ = si.to_bf16(si.bases(8202, 1, Hkv * d, rV)[0])
    k_lat = torch.zeros((B, Hkv, L_max, rK), dtype=torch.bfloat16, device=DEV)
    v_joint = torch.zeros((B, L_max, rV), dtype=torch.bfloat16, device=DEV)
    lens = torch.tensor([0, 40], dtype=torch.int32, device=DEV)
    status = torch.zeros(1, dtype=torch.int32, device=DEV)
    wk, wv = np.zeros((B, Hkv, L_max, rK)), np.zeros((B, L_max, rV))
    wl = np.array([0, 40], np.int32)
    for kk, vv in ((k_pre, v_pre), (k_new, v_new)):
        stief.stief_compress_append_joint_v(kk.to(DEV), vv.to(DEV), P_K.to(DEV), P_VJ.to(DEV),
                                            k_lat, v_joint, lens, dev_status=status)
        wk, wv, wl, _ = oracle.compress_append_joint_v(f64(kk), f64(vv), f64(P_K), f64(P_VJ),
                                                       wk, wv, wl)
    assert stief.stief_read_device_status(status) == 0
    assert lens.cpu().tolist() == wl.tolist() == [151, 191]
    q = si.queries(8203, B, Hq, d)
    got = _gpu_joint(q, P_K, P_VJ, k_lat, v_joint, wl.tolist(), max_seq_len=L_max)
    assert_decode_close(got, oracle.decode_joint_v(f64(q), f64(P_K), f64(P_VJ), wk, wv, wl))


# ------------------------------------------------- joint compress, prefill-sized chunks (tcgen05)

def _check_within_fp32_bound(k_new, v_new, P_K, P_VJ, gk, gv, lens):
    """Every stored row against the exact products: within half a bf16 ulp plus the fp32
    accumulation bound K * 2^-23 * sum|x||p| (K = d for the keys, Hkv*d for the values)."""
    B, Hkv, T, d = k_new.shape
    P = f64(P_VJ)
    for b, L in enumerate(lens):
        x = np.ascontiguousarray(np.transpose(f64(v_new[b]), (1, 0, 2)).reshape(T, Hkv * d))
        exact = x @ P
        bound = 2.0 ** -8 * np.abs(exact) + Hkv * d * 2.0 ** -23 * (np.abs(x) @ np.abs(P)) + 1e-30
        assert np.all(np.abs(f64(gv[b, L:L + T]) - exact) <= bound)
        for h in range(Hkv):
            xk, pk = f64(k_new[b, h]), f64(P_K[h])
            ek = xk @ pk
            kb = 2.0 ** -8 * np.abs(ek) + d * 2.0 ** -23 * (np.abs(xk) @ np.abs(pk)) + 1e-30
            assert np.all(np.abs(f64(gk[b, h, L:L + T]) - ek) <= kb)


@pytest.mark.parametrize("T", [128, 129, 300, 1000])
def test_compress_tc_selector_bases_bit_exact(T):
    """Chunks of 128 rows or more take the tensor-core projection: with selector bases every
    stored value is one input coordinate, bit for bit the oracle's, at the rows the lengths
    name, nothing written elsewhere (ragged last tiles included)."""
    B, Hkv, d, rK, rV = 2, 4, 128, 32, 48
    L_max = T + 40
    k_new, v_new = si.full_kv(8300 + T, B, Hkv, T, d)
    P_K = torch.stack([_selector_basis(1, d, rK) for _ in range(Hkv)])
    P_VJ = _selector_basis(Hkv, d, rV)
    lens = [0, 37]
    gk, gv, glens, st = _compress_joint(k_new, v_new, P_K, P_VJ, L_max, lens)
    assert st == 0 and glens.tolist() == [L + T for L in lens]
    wk, wv, wl, nbad = oracle.compress_append_joint_v(
        f64(k_new), f64(v_new), f64(P_K), f64(P_VJ), np.zeros((B, Hkv, L_max, rK)),
        np.zeros((B, L_max, rV)), np.asarray(lens, np.int32))
    assert nbad == 0 and wl.tolist() == glens.tolist()
    for b, L in enumerate(lens):
        assert np.array_equal(f64(gk[b, :, L:L + T]), wk[b, :, L:L + T])
        assert np.array_equal(f64(gv[b, L:L + T]), wv[b, L:L + T])
        keep = np.ones(L_max, bool)
        keep[L:L + T] = False
        assert torch.all(gk[b][:, keep].view(torch.int16) == CANARY)
        assert torch.all(gv[b][keep].view(torch.int16) == CANARY)


@pytest.mark.parametrize("B,Hkv,T,rK,rV", [
    (1, 8, 4096, 64, 64),    # one prefill chunk of the 8B-class models (K = 1024 for the values)
    (1, 8, 4096, 32, 48),
    (2, 2, 10240, 64, 64),   # several tiles per CTA, the ring wrapping many times
    (1, 1, 1153, 128, 128),  # one KV head, the widest ranks, a ragged tail
    (3, 4, 640, 16, 112),
    (1, 8, 256, 64, 128),    # the joint basis (256 KB) does not fit: the CUDA-core projection
])
def test_compress_tc_general_bases_within_the_fp32_bound(B, Hkv, T, rK, rV):
    """General bases at prefill sizes: every stored key and joint value row within the fp32
    bound of the exact product, lengths advanced, and (as a check on the accumulation
    order only) almost every row equal to the oracle's bf16 rounding."""
    d = 128
    lens = [5 + 17 * b for b in range(B)]
    L_max = T + 64
    k_new, v_new = si.full_kv(8400 + T + Hkv, B, Hkv, T, d)
    P_K = si.to_bf16(si.bases(8400 + rK, Hkv, d, rK))
    P_VJ = si.to_bf16(si.bases(8401 + rV, 1, Hkv * d, rV)[0])
    gk, gv, glens, st = _compress_joint(k_new, v_new, P_K, P_VJ, L_max, lens)
    assert st == 0 and glens.tolist() == [L + T for L in lens]
    _check_within_fp32_bound(k_new, v_new, P_K, P_VJ, gk, gv, lens)
    want = oracle.compress_append_joint_v(f64(k_new), f64(v_new), f64(P_K), f64(P_VJ),
                                          np.zeros((B, Hkv, L_max, rK)), np.zeros((B, L_max, rV)),
                                          np.asarray(lens, np.int32))[1]
    same = [np.mean(f64(gv[b, L:L + T]) == want[b, L:L + T]) for b, L in enumerate(lens)]
    assert min(same) > 0.95
    for b, L in enumerate(lens):
        keep = np.ones(L_max, bool)
        keep[L:L + T] = False
        assert torch.all(gv[b][keep].view(torch.int16) == CANARY)
        assert torch.all(gk[b][:, keep].view(torch.int16) == CANARY)


def test_compress_tc_refuses_full_and_bad_sequences():
    """On the tensor-core path too: a sequence with no room for the chunk and one with a
    negative length are skipped (nothing written, length unchanged) and reported; the
    others are appended."""
    B, Hkv, d, rK, rV, T = 3, 8, 128, 64, 64, 200
    L_max = 300
    k_new, v_new = si.full_kv(8500, B, Hkv, T, d)
    P_K = si.to_bf16(si.bases(8500, Hkv, d, rK))
    P_VJ = si.to_bf16(si.bases(8501, 1, Hkv * d, rV)[0])
    lens = [L_max - T + 1, -1, L_max - T]
    gk, gv, glens, st = _compress_joint(k_new, v_new, P_K, P_VJ, L_max, lens)
    assert st == (stief.DEV_CAPACITY_OVERFLOW | stief.DEV_BAD_LENGTH)
    assert glens.tolist() == [lens[0], -1, L_max]
    for b in (0, 1):
        assert torch.all(gk[b].view(torch.int16) == CANARY)
        assert torch.all(gv[b].view(torch.int16) == CANARY)
    _check_within_fp32_bound(k_new[2:], v_new[2:], P_K, P_VJ, gk[2:], gv[2:], [lens[2]])


def test_compress_tc_then_decode_same_stream():
    """A 2048-token joint chunk compressed and decoded right after it on the same stream (the
    compress's length kernel lets the decode start early; the decode must still see the new
    rows and lengths), against the oracle's joint compress and decode."""
    B, Hq, Hkv, d, rK, rV, T = 2, 32, 8, 128, 64, 64, 2048
    L_max = T + 64
    k_new, v_new = si.full_kv(8600, B, Hkv, T, d)
    P_K = si.to_bf16(si.bases(8600, Hkv, d, rK))
    P_VJ = si.to_bf16(si.bases(8602, 1, Hkv * d, rV)[0])
    q = si.queries(8603, B, Hq, d)
    k_lat = torch.zeros((B, Hkv, L_max, rK), dtype=torch.bfloat16, device=DEV)
    v_joint = torch.zeros((B, L_max, rV), dtype=torch.bfloat16, device=DEV)
    lens0 = [3, 60]
    lens = torch.tensor(lens0, dtype=torch.int32, device=DEV)
    qd, P_Kd, P_VJd = q.to(DEV), P_K.to(DEV), P_VJ.to(DEV)
    out = torch.empty((B, Hq, d), dtype=torch.bfloat16, device=DEV)
    ws = _ws(B, Hq, Hkv, rV, L_max)
    status = torch.zeros(1, dtype=torch.int32, device=DEV)
    stief.stief_compress_append_joint_v(k_new.to(DEV), v_new.to(DEV), P_Kd, P_VJd, k_lat, v_joint,
                                        lens, dev_status=status)
    stief.stief_decode_attention_joint_v(qd, P_Kd, P_VJd, k_lat, v_joint, lens, out, ws,
                                         max_seq_len=L_max, dev_status=status)
    torch.cuda.synchronize()
    assert stief.stief_read_device_status(status) == 0
    wk, wv, wl, _ = oracle.compress_append_joint_v(
        f64(k_new), f64(v_new), f64(P_K), f64(P_VJ), f64(k_lat.cpu()) * 0, f64(v_joint.cpu()) * 0,
        np.asarray(lens0, np.int32))
    assert lens.cpu().tolist() == wl.tolist()
    # the decode reads the GPU's stored rows: compare it with the oracle on those rows, and the
    # rows with the oracle's compress within the accumulation bound
    _check_within_fp32_bound(k_new, v_new, P_K, P_VJ, k_lat.cpu(), v_joint.cpu(), lens0)
    want = oracle.decode_joint_v(f64(q), f64(P_K), f64(P_VJ), f64(k_lat.cpu()), f64(v_joint.cpu()), wl)
    assert_decode_close(out.cpu(), want)
