"""4-bit latent caches: stief_compress_append_q4 and stief_decode_attention_q4 (CUDA, through
the C ABI) against the fp64 oracle.

The stored form is the oracle's quantize_rows with qmax = 7 (one fp32 scale per row, RNE codes
in [-7, 7], both divisions in IEEE fp32) applied to the bf16-rounded latent row, packed two
codes per byte by pack_q4 (column 2j in the low nibble of byte j).  With the identity basis
the latent rows are exact bf16 values on both sides, so the packed bytes and the scales must
be bit-identical; with general bases the GPU's bf16 row can differ from the oracle's by an
ulp at a rounding boundary, so codes may differ by one there.  The decode is checked against
the oracle's decode over code * scale, tolerance 2e-2 * ||o||_inf as for the bf16 cache.
"""
import numpy as np
import pytest
import torch

import decode_attention_stief_b200 as stief
import oracle
import stief_inputs as si
from gpu_util import assert_decode_close, f64

pytestmark = pytest.mark.gpu
DEV = torch.device("cuda")


def _identity_basis(Hkv, d, r):
    P = np.zeros((Hkv, d, r))
    for h in range(Hkv):
        P[h, :r, :] = np.eye(r)
    return si.to_bf16(P)


def _compress_q4(k_new, v_new, P_K, P_V, B, Hkv, L_max, rK, rV, lens, expect_status=0):
    kq = torch.zeros((B, Hkv, L_max, rK // 2), dtype=torch.uint8, device=DEV)
    vq = torch.zeros((B, Hkv, L_max, rV // 2), dtype=torch.uint8, device=DEV)
    ks = torch.zeros((B, Hkv, L_max), dtype=torch.float32, device=DEV)
    vs = torch.zeros((B, Hkv, L_max), dtype=torch.float32, device=DEV)
    glens = torch.as_tensor(np.asarray(lens, np.int32)).to(DEV)
    status = torch.zeros(1, dtype=torch.int32, device=DEV)
    stief.stief_compress_append_q4(k_new.to(DEV), v_new.to(DEV), P_K.to(DEV), P_V.to(DEV), kq, vq,
                                   ks, vs, glens, dev_status=status)
    assert stief.stief_read_device_status(status) == expect_status
    return kq.cpu(), vq.cpu(), ks.cpu(), vs.cpu(), glens.cpu().numpy()


def _random_q4_cache(seed, B, Hkv, L, r):
    """Seeded packed codes and scales: the 4-bit form of a low-rank latent cache."""
    lat = si.latent_cache(seed, B, Hkv, L, r, 0)
    q, s = oracle.quantize_rows(f64(lat), qmax=7)
    return torch.from_numpy(oracle.pack_q4(q)), torch.from_numpy(s)


def _deq(packed, scales):
    return oracle.dequantize_rows(oracle.unpack_q4(packed.numpy()), scales.numpy())


def _decode_q4(q, P_K, P_V, kq, vq, ks, vs, lens, max_seq_len, num_splits=0):
    B, Hq, d = q.shape
    out = torch.full((B, Hq, d), float("nan"), dtype=torch.bfloat16, device=DEV)
    ws = stief.workspace_for(B, Hq, P_K.shape[0], P_V.shape[2], max_seq_len)
    status = torch.zeros(1, dtype=torch.int32, device=DEV)
    stief.stief_decode_attention_q4(q.to(DEV), P_K.to(DEV), P_V.to(DEV), kq.to(DEV), vq.to(DEV),
                                    ks.to(DEV), vs.to(DEV),
                                    torch.as_tensor(np.asarray(lens, np.int32)).to(DEV), out, ws,
                                    max_seq_len, num_splits=num_splits, dev_status=status)
    assert stief.stief_read_device_status(status) == 0
    return out.cpu()


def _case(seed, B, Hq, Hkv, L, rK, rV, q_scale=1.0):
    q = si.queries(seed, B, Hq, 128, scale=q_scale)
    P_K, P_V = si.bases_bf16(seed + 1, Hkv, 128, rK, rV)
    kq, ks = _random_q4_cache(seed + 2, B, Hkv, L, rK)
    vq, vs = _random_q4_cache(seed + 3, B, Hkv, L, rV)
    return q, P_K, P_V, kq, vq, ks, vs


def _oracle(q, P_K, P_V, kq, vq, ks, vs, lens):
    return oracle.decode(f64(q), f64(P_K), f64(P_V), _deq(kq, ks), _deq(vq, vs),
                         np.asarray(lens, np.int32))


@pytest.mark.parametrize("T", [1, 5, 8, 200])
def test_identity_basis_codes_and_scales_are_bit_exact(T):
    """Both compress paths (CUDA cores for T < 128, tensor cores for T >= 128)."""
    B, Hkv, rK, rV, L_max = 2, 2, 64, 32, 256
    k_new, v_new = si.full_kv(7100 + T, B, Hkv, T, 128)
    P_K, P_V = _identity_basis(Hkv, 128, rK), _identity_basis(Hkv, 128, rV)
    lens = [3, 40]
    kq, vq, ks, vs, glens = _compress_q4(k_new, v_new, P_K, P_V, B, Hkv, L_max, rK, rV, lens)
    assert glens.tolist() == [3 + T, 40 + T]
    for b in range(B):
        wk, wks = oracle.quantize_rows(f64(k_new[b])[..., :rK], qmax=7)
        wv, wvs = oracle.quantize_rows(f64(v_new[b])[..., :rV], qmax=7)
        sl = slice(lens[b], lens[b] + T)
        assert np.array_equal(kq[b, :, sl].numpy(), oracle.pack_q4(wk))
        assert np.array_equal(vq[b, :, sl].numpy(), oracle.pack_q4(wv))
        assert np.array_equal(ks[b, :, sl].numpy(), wks)
        assert np.array_equal(vs[b, :, sl].numpy(), wvs)
        # rows outside the appended range are untouched
        assert torch.all(kq[b, :, :lens[b]] == 0) and torch.all(kq[b, :, lens[b] + T:] == 0)


@pytest.mark.parametrize("T", [3, 130])
def test_general_bases_codes_within_one(T):
    B, Hkv, rK, rV, L_max = 1, 4, 64, 64, 192
    k_new, v_new = si.full_kv(7200 + T, B, Hkv, T, 128)
    P_K, P_V = si.bases_bf16(7200 + T, Hkv, 128, rK, rV)
    kq, vq, ks, vs, _ = _compress_q4(k_new, v_new, P_K, P_V, B, Hkv, L_max, rK, rV, [10])
    for h in range(Hkv):
        lat = oracle.project(f64(k_new[0, h]), f64(P_K[h]))
        wq, wsc = oracle.quantize_rows(lat, qmax=7)
        got = oracle.unpack_q4(kq[0, h, 10:10 + T].numpy()).astype(int)
        assert np.max(np.abs(got - wq)) <= 1
        assert np.allclose(ks[0, h, 10:10 + T].numpy(), wsc, rtol=2e-2)


@pytest.mark.parametrize("rK,rV", [(64, 64), (32, 32), (96, 128), (32, 64), (128, 32)])
@pytest.mark.parametrize("num_splits", [0, 1, 3])
def test_decode_q4_matches_oracle(rK, rV, num_splits):
    B, Hq, Hkv, L = 3, 16, 4, 704
    lens = [700, 33, 0]
    args = _case(7300 + rK + rV, B, Hq, Hkv, L, rK, rV)
    got = _decode_q4(*args, lens, 700, num_splits)
    assert_decode_close(got, _oracle(*args, lens))
    assert torch.all(got[2].float() == 0)


@pytest.mark.parametrize("Hq,Hkv", [(32, 4), (8, 4), (24, 4), (4, 4)])
def test_decode_q4_group_sizes(Hq, Hkv):
    B, L, rK, rV = 2, 448, 64, 64
    lens = [445, 130]
    args = _case(7400 + Hq, B, Hq, Hkv, L, rK, rV)
    got = _decode_q4(*args, lens, 445, 2)
    assert_decode_close(got, _oracle(*args, lens))


@pytest.mark.parametrize("lens", [[63, 64, 65], [1, 31, 32]])
def test_decode_q4_tile_boundaries(lens):
    B, Hq, Hkv, L, rK, rV = 3, 16, 4, 192, 64, 64
    args = _case(7500 + sum(lens), B, Hq, Hkv, L, rK, rV)
    got = _decode_q4(*args, lens, 65, 0)
    assert_decode_close(got, _oracle(*args, lens))


def test_decode_q4_peaked_scores():
    B, Hq, Hkv, L, rK, rV = 2, 32, 8, 1024, 64, 64
    lens = [1024, 517]
    args = _case(7600, B, Hq, Hkv, L, rK, rV, q_scale=8.0)
    got = _decode_q4(*args, lens, 1024, 0)
    assert_decode_close(got, _oracle(*args, lens))


def test_decode_q4_rows_past_length_hold_garbage():
    B, Hq, Hkv, L, rK, rV = 3, 16, 4, 384, 32, 64
    lens = [300, 33, 0]
    q, P_K, P_V, kq, vq, ks, vs = _case(7700, B, Hq, Hkv, L, rK, rV)
    kq, vq, ks, vs = kq.clone(), vq.clone(), ks.clone(), vs.clone()
    rng = np.random.default_rng(7701)
    bad = np.array([np.nan, np.inf, -np.inf, 3e38], np.float32)
    for b in range(B):
        n = L - lens[b]
        kq[b, :, lens[b]:] = torch.from_numpy(rng.integers(0, 256, (Hkv, n, rK // 2), dtype=np.uint8))
        vq[b, :, lens[b]:] = torch.from_numpy(rng.integers(0, 256, (Hkv, n, rV // 2), dtype=np.uint8))
        ks[b, :, lens[b]:] = torch.from_numpy(rng.choice(bad, (Hkv, n)))
        vs[b, :, lens[b]:] = torch.from_numpy(rng.choice(bad, (Hkv, n)))
    got = _decode_q4(q, P_K, P_V, kq, vq, ks, vs, lens, 384, 3)
    want = oracle.decode(f64(q), f64(P_K), f64(P_V),
                         _deq(kq, torch.nan_to_num(ks, 0.0, 0.0, 0.0)),
                         _deq(vq, torch.nan_to_num(vs, 0.0, 0.0, 0.0)), np.asarray(lens, np.int32))
    assert_decode_close(got, want)
    assert torch.all(got[2].float() == 0)


def test_compress_then_decode_q4_end_to_end():
    B, Hq, Hkv, rK, rV, T, L_max = 2, 32, 8, 64, 32, 300, 320
    k_new, v_new = si.full_kv(7800, B, Hkv, T, 128)
    P_K, P_V = si.bases_bf16(7800, Hkv, 128, rK, rV)
    kq, vq, ks, vs, glens = _compress_q4(k_new, v_new, P_K, P_V, B, Hkv, L_max, rK, rV, [0, 0])
    q = si.queries(7801, B, Hq, 128)
    lens = [300, 171]
    got = _decode_q4(q, P_K, P_V, kq, vq, ks, vs, lens, L_max)
    wk = np.zeros((B, Hkv, L_max, rK))
    wv = np.zeros((B, Hkv, L_max, rV))
    for b in range(B):
        for h in range(Hkv):
            c, s = oracle.quantize_rows(oracle.project(f64(k_new[b, h]), f64(P_K[h])), qmax=7)
            wk[b, h, :T] = oracle.dequantize_rows(c, s)
            c, s = oracle.quantize_rows(oracle.project(f64(v_new[b, h]), f64(P_V[h])), qmax=7)
            wv[b, h, :T] = oracle.dequantize_rows(c, s)
    want = oracle.decode(f64(q), f64(P_K), f64(P_V), wk, wv, np.asarray(lens, np.int32))
    assert_decode_close(got, want)


def test_decode_q4_full_size_32k():
    """The 32k benchmark shape at full context over a 4-bit cache."""
    w = si.WORKLOADS["llama3_8b_32k"]
    seed = si.sub_seed(w.seed, 49)
    k = si.latent_cache_torch(seed, w.B, w.Hkv, w.L, w.rK, 0, DEV)
    v = si.latent_cache_torch(seed, w.B, w.Hkv, w.L, w.rV, 1, DEV)
    kc, ks = oracle.quantize_rows(f64(k), qmax=7)
    vc, vs = oracle.quantize_rows(f64(v), qmax=7)
    kq, vq = torch.from_numpy(oracle.pack_q4(kc)), torch.from_numpy(oracle.pack_q4(vc))
    ks, vs = torch.from_numpy(ks), torch.from_numpy(vs)
    q = si.queries_torch(seed + 1, w.B, w.Hq, w.d, DEV)
    P_K, P_V = si.bases_bf16(seed, w.Hkv, w.d, w.rK, w.rV)
    got = _decode_q4(q, P_K, P_V, kq, vq, ks, vs, [w.L] * w.B, w.L)
    want = oracle.decode(f64(q), f64(P_K), f64(P_V), oracle.dequantize_rows(kc, ks.numpy()),
                         oracle.dequantize_rows(vc, vs.numpy()), np.full(w.B, w.L, np.int32))
    assert_decode_close(got, want)


def test_decode_q4_multi_wave_grid():
    B, Hq, Hkv, rK, rV, L = 40, 32, 8, 64, 64, 320
    rng = np.random.default_rng(7900)
    lens = rng.integers(1, L, size=B).tolist()
    lens[5] = 0
    lens[9] = L
    args = _case(7900, B, Hq, Hkv, L, rK, rV)
    got = _decode_q4(*args, lens, L)
    assert_decode_close(got, _oracle(*args, lens))
    assert torch.all(got[5].float() == 0)


def test_q4_rejects_ranks_not_multiple_of_32():
    B, Hq, Hkv, L = 1, 8, 2, 128
    q, P_K, P_V, kq, vq, ks, vs = _case(8000, B, Hq, Hkv, L, 32, 32)
    P_K48 = si.bases_bf16(8000, Hkv, 128, 48, 32)[0]
    kq48 = torch.zeros((B, Hkv, L, 24), dtype=torch.uint8)
    with pytest.raises(stief.StiefError):
        _decode_q4(q, P_K48, P_V, kq48, vq, ks, vs, [10], L)
