"""int8 latent caches: stief_compress_append_q8 and stief_decode_attention_q8 (CUDA, through
the C ABI) against the fp64 oracle.

The stored form is the oracle's quantize_rows (one fp32 scale per row, RNE codes, both
divisions in IEEE fp32) applied to the bf16-rounded latent row.  With the identity basis the
latent rows are exact bf16 values on both sides, so the integer codes and the scales must be
bit-identical; with general bases the GPU's bf16 row can differ from the oracle's by an ulp
at a rounding boundary, so codes may differ by one there.  The decode is checked against
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


def _compress_q8(k_new, v_new, P_K, P_V, B, Hkv, L_max, rK, rV, lens, expect_status=0):
    kq = torch.zeros((B, Hkv, L_max, rK), dtype=torch.int8, device=DEV)
    vq = torch.zeros((B, Hkv, L_max, rV), dtype=torch.int8, device=DEV)
    ks = torch.full((B, Hkv, L_max), -1.0, dtype=torch.float32, device=DEV)
    vs = torch.full((B, Hkv, L_max), -1.0, dtype=torch.float32, device=DEV)
    lens_t = torch.as_tensor(np.asarray(lens, np.int32)).to(DEV)
    status = torch.zeros(1, dtype=torch.int32, device=DEV)
    stief.stief_compress_append_q8(k_new.to(DEV), v_new.to(DEV), P_K.to(DEV), P_V.to(DEV), kq, vq,
                                   ks, vs, lens_t, dev_status=status)
    assert stief.stief_read_device_status(status) == expect_status
    return kq.cpu(), vq.cpu(), ks.cpu(), vs.cpu(), lens_t.cpu().numpy()


@pytest.mark.parametrize("T", [1, 5, 8, 200])
def test_identity_basis_codes_and_scales_are_bit_exact(T):
    """P = [I; 0]: the latent row is the first r coordinates of the bf16 row exactly, so the
    quantisation decisions are taken on identical inputs (CUDA-core path T < 128, tensor
    cores from 128)."""
    B, Hkv, rK, rV, L_max = 2, 2, 64, 48, 256
    k_new, v_new = si.full_kv(6000 + T, B, Hkv, T, 128)
    P_K, P_V = _identity_basis(Hkv, 128, rK), _identity_basis(Hkv, 128, rV)
    lens = [0, 37]
    kq, vq, ks, vs, glens = _compress_q8(k_new, v_new, P_K, P_V, B, Hkv, L_max, rK, rV, lens)
    assert glens.tolist() == [L + T for L in lens]
    for b, L in enumerate(lens):
        wk, wks = oracle.quantize_rows(f64(k_new[b])[..., :rK])
        wv, wvs = oracle.quantize_rows(f64(v_new[b])[..., :rV])
        assert np.array_equal(kq[b, :, L:L + T].numpy(), wk)
        assert np.array_equal(vq[b, :, L:L + T].numpy(), wv)
        assert np.array_equal(ks[b, :, L:L + T].numpy(), wks)
        assert np.array_equal(vs[b, :, L:L + T].numpy(), wvs)
        assert torch.all(ks[b, :, :L] == -1) and torch.all(ks[b, :, L + T:] == -1)


@pytest.mark.parametrize("T", [3, 130])
def test_general_bases_codes_within_one(T):
    B, Hkv, rK, rV, L_max = 1, 4, 64, 64, 192
    k_new, v_new = si.full_kv(6100 + T, B, Hkv, T, 128)
    P_K, P_V = si.bases_bf16(6100 + T, Hkv, 128, rK, rV)
    kq, vq, ks, vs, _ = _compress_q8(k_new, v_new, P_K, P_V, B, Hkv, L_max, rK, rV, [10])
    for m, (q, s, x, P) in enumerate(((kq, ks, k_new, P_K), (vq, vs, v_new, P_V))):
        for h in range(Hkv):
            lat = oracle.project(f64(x[0, h]), f64(P[h]), round_to_bf16=True)
            wq, ws = oracle.quantize_rows(lat)
            gq = q[0, h, 10:10 + T].numpy().astype(np.int32)
            assert np.max(np.abs(gq - wq.astype(np.int32))) <= 1
            assert np.mean(gq == wq) > 0.98
            np.testing.assert_allclose(s[0, h, 10:10 + T].numpy(), ws, rtol=2 ** -7)


def _random_q8_cache(seed, B, Hkv, L, r):
    """Seeded codes and scales: the int8 form of a low-rank latent cache."""
    lat = si.latent_cache(seed, B, Hkv, L, r, 0)
    q, s = oracle.quantize_rows(f64(lat))
    return torch.from_numpy(q), torch.from_numpy(s)


def _decode_q8(q, P_K, P_V, kq, vq, ks, vs, lens, max_seq_len, num_splits=0):
    B, Hq, d = q.shape
    out = torch.full((B, Hq, d), float("nan"), dtype=torch.bfloat16, device=DEV)
    ws = stief.workspace_for(B, Hq, P_K.shape[0], P_V.shape[2], max_seq_len)
    status = torch.zeros(1, dtype=torch.int32, device=DEV)
    stief.stief_decode_attention_q8(q.to(DEV), P_K.to(DEV), P_V.to(DEV), kq.to(DEV), vq.to(DEV),
                                    ks.to(DEV), vs.to(DEV),
                                    torch.as_tensor(np.asarray(lens, np.int32)).to(DEV), out, ws,
                                    max_seq_len, num_splits=num_splits, dev_status=status)
    assert stief.stief_read_device_status(status) == 0
    return out.cpu()


@pytest.mark.parametrize("rK,rV", [(64, 64), (32, 48), (96, 128), (16, 16)])
@pytest.mark.parametrize("num_splits", [0, 1, 3])
def test_decode_q8_matches_oracle(rK, rV, num_splits):
    B, Hq, Hkv, L = 3, 16, 4, 704
    lens = [700, 33, 0]
    q = si.queries(6200 + rK, B, Hq, 128)
    P_K, P_V = si.bases_bf16(6200 + rV, Hkv, 128, rK, rV)
    kq, ks = _random_q8_cache(6201 + rK, B, Hkv, L, rK)
    vq, vs = _random_q8_cache(6202 + rV, B, Hkv, L, rV)
    got = _decode_q8(q, P_K, P_V, kq, vq, ks, vs, lens, 700, num_splits)
    want = oracle.decode(f64(q), f64(P_K), f64(P_V), oracle.dequantize_rows(kq.numpy(), ks.numpy()),
                         oracle.dequantize_rows(vq.numpy(), vs.numpy()), np.asarray(lens, np.int32))
    assert_decode_close(got, want)
    assert torch.all(got[2].float() == 0)


def test_compress_then_decode_q8_end_to_end():
    """Prefill chunk into an int8 cache on the tensor cores, then a decode over it, against
    the oracle's projection, quantisation and decode."""
    B, Hq, Hkv, rK, rV, T, L_max = 2, 32, 8, 64, 64, 300, 320
    k_new, v_new = si.full_kv(6300, B, Hkv, T, 128)
    P_K, P_V = si.bases_bf16(6300, Hkv, 128, rK, rV)
    kq, vq, ks, vs, glens = _compress_q8(k_new, v_new, P_K, P_V, B, Hkv, L_max, rK, rV, [0, 0])
    q = si.queries(6301, B, Hq, 128)
    lens = [300, 171]
    got = _decode_q8(q, P_K, P_V, kq, vq, ks, vs, lens, L_max)
    wk = np.zeros((B, Hkv, L_max, rK))
    wv = np.zeros((B, Hkv, L_max, rV))
    for b in range(B):
        for h in range(Hkv):
            c, s = oracle.quantize_rows(oracle.project(f64(k_new[b, h]), f64(P_K[h])))
            wk[b, h, :T] = oracle.dequantize_rows(c, s)
            c, s = oracle.quantize_rows(oracle.project(f64(v_new[b, h]), f64(P_V[h])))
            wv[b, h, :T] = oracle.dequantize_rows(c, s)
    want = oracle.decode(f64(q), f64(P_K), f64(P_V), wk, wv, np.asarray(lens, np.int32))
    assert_decode_close(got, want)


@pytest.mark.parametrize("name", ["llama3_8b_32k", "llama31_8b_128k"])
def test_decode_q8_full_size(name):
    """The benchmark shapes at full context over an int8 cache; sequence 0 checked exactly."""
    w = si.WORKLOADS[name]
    seed = si.sub_seed(w.seed, 48)
    k = si.latent_cache_torch(seed, w.B, w.Hkv, w.L, w.rK, 0, DEV)
    v = si.latent_cache_torch(seed, w.B, w.Hkv, w.L, w.rV, 1, DEV)
    kq, ks = oracle.quantize_rows(f64(k))
    vq, vs = oracle.quantize_rows(f64(v))
    kq, ks, vq, vs = (torch.from_numpy(x) for x in (kq, ks, vq, vs))
    q = si.queries_torch(seed + 1, w.B, w.Hq, w.d, DEV)
    P_K, P_V = si.bases_bf16(seed, w.Hkv, w.d, w.rK, w.rV)
    got = _decode_q8(q, P_K, P_V, kq, vq, ks, vs, [w.L] * w.B, w.L)
    want = oracle.decode(f64(q), f64(P_K), f64(P_V), oracle.dequantize_rows(kq.numpy(), ks.numpy()),
                         oracle.dequantize_rows(vq.numpy(), vs.numpy()), np.full(w.B, w.L, np.int32))
    assert_decode_close(got, want)


def test_decode_q8_multi_wave_grid():
    """More units than SMs (40 x 8 = 320): the int8 decode in the two-CTAs-per-SM plan."""
    B, Hq, Hkv, rK, rV, L = 40, 32, 8, 64, 64, 320
    rng = np.random.default_rng(6400)
    lens = rng.integers(1, L, size=B).tolist()
    lens[5] = 0
    lens[9] = L
    q = si.queries(6400, B, Hq, 128)
    P_K, P_V = si.bases_bf16(6400, Hkv, 128, rK, rV)
    kq, ks = _random_q8_cache(6401, B, Hkv, L, rK)
    vq, vs = _random_q8_cache(6402, B, Hkv, L, rV)
    got = _decode_q8(q, P_K, P_V, kq, vq, ks, vs, lens, L)
    want = oracle.decode(f64(q), f64(P_K), f64(P_V), oracle.dequantize_rows(kq.numpy(), ks.numpy()),
                         oracle.dequantize_rows(vq.numpy(), vs.numpy()), np.asarray(lens, np.int32))
    assert_decode_close(got, want)
    assert torch.all(got[5].float() == 0)


def _q8_case(seed, B, Hq, Hkv, L, rK, rV, q_scale=1.0):
    q = si.queries(seed, B, Hq, 128, scale=q_scale)
    P_K, P_V = si.bases_bf16(seed + 1, Hkv, 128, rK, rV)
    kq, ks = _random_q8_cache(seed + 2, B, Hkv, L, rK)
    vq, vs = _random_q8_cache(seed + 3, B, Hkv, L, rV)
    return q, P_K, P_V, kq, vq, ks, vs


def _oracle_q8(q, P_K, P_V, kq, vq, ks, vs, lens):
    return oracle.decode(f64(q), f64(P_K), f64(P_V), oracle.dequantize_rows(kq.numpy(), ks.numpy()),
                         oracle.dequantize_rows(vq.numpy(), vs.numpy()), np.asarray(lens, np.int32))


@pytest.mark.parametrize("Hq,Hkv", [(32, 4), (8, 4), (24, 4), (4, 4)])
@pytest.mark.parametrize("num_splits", [0, 2])
def test_decode_q8_group_sizes(Hq, Hkv, num_splits):
    """Query groups of 8 (the hi and lo parts in two n-tiles), 2, 6 (padded to 8) and 1."""
    B, L, rK, rV = 2, 448, 64, 64
    lens = [445, 130]
    args = _q8_case(6500 + Hq, B, Hq, Hkv, L, rK, rV)
    got = _decode_q8(*args, lens, 445, num_splits)
    assert_decode_close(got, _oracle_q8(*args, lens))


@pytest.mark.parametrize("rK,rV", [(48, 16), (80, 112), (112, 48), (16, 96), (128, 128)])
def test_decode_q8_odd_ranks(rK, rV):
    """Ranks whose rows are 16 x odd bytes: a 16-code last k-step for the scores, and 16-byte
    (unswizzled) column pieces for the values and keys."""
    B, Hq, Hkv, L = 2, 16, 4, 320
    lens = [317, 64]
    args = _q8_case(6600 + rK + rV, B, Hq, Hkv, L, rK, rV)
    got = _decode_q8(*args, lens, 317, 0)
    assert_decode_close(got, _oracle_q8(*args, lens))


@pytest.mark.parametrize("lens", [[63, 64, 65], [127, 128, 129], [1, 31, 32]])
def test_decode_q8_tile_boundaries(lens):
    """Lengths at the 32- and 64-token tile edges (the 64/64 ranks take 64-token tiles)."""
    B, Hq, Hkv, L, rK, rV = 3, 16, 4, 192, 64, 64
    args = _q8_case(6700 + sum(lens), B, Hq, Hkv, L, rK, rV)
    got = _decode_q8(*args, lens, 129, 0)
    assert_decode_close(got, _oracle_q8(*args, lens))


@pytest.mark.parametrize("q_scale", [4.0, 16.0])
def test_decode_q8_peaked_scores(q_scale):
    """Large queries make the softmax peaked (a few tokens carry the weight; the running
    maximum is rescaled often)."""
    B, Hq, Hkv, L, rK, rV = 2, 32, 8, 1024, 64, 64
    lens = [1024, 517]
    args = _q8_case(6800, B, Hq, Hkv, L, rK, rV, q_scale=q_scale)
    got = _decode_q8(*args, lens, 1024, 0)
    assert_decode_close(got, _oracle_q8(*args, lens))


def test_decode_q8_needle_and_spread_mass():
    """One needle token per (sequence, KV head) whose score is 12 above the other tokens' best,
    so that it carries most of the weight while the rest still hold a few per cent: the
    per-tile fixed point of the weights must keep both."""
    B, Hq, Hkv, L, rK, rV = 2, 16, 4, 2048, 64, 64
    G = Hq // Hkv
    lens = [2048, 1500]
    q, P_K, P_V, kq, vq, ks, vs = _q8_case(6900, B, Hq, Hkv, L, rK, rV)
    kq, ks = kq.clone(), ks.clone()
    rng = np.random.default_rng(6901)
    k_deq = oracle.dequantize_rows(kq.numpy(), ks.numpy())
    for b in range(B):
        for h in range(Hkv):
            qt = f64(q[b, h * G]) @ f64(P_K[h])  # q~ of the group's first head
            s = k_deq[b, h, :lens[b]] @ qt / np.sqrt(128.0)
            pos = int(rng.integers(0, lens[b]))
            codes = np.where(qt >= 0, 127, -127).astype(np.int8)
            scale = (s.max() + 12.0) * np.sqrt(128.0) / (127.0 * np.abs(qt).sum())
            kq[b, h, pos] = torch.from_numpy(codes)
            ks[b, h, pos] = float(np.float32(scale))
    args = (q, P_K, P_V, kq, vq, ks, vs)
    got = _decode_q8(*args, lens, 2048, 0)
    assert_decode_close(got, _oracle_q8(*args, lens))


@pytest.mark.parametrize("num_splits", [0, 3])
def test_decode_q8_rows_past_length_hold_garbage(num_splits):
    """Codes and scales past each length are arbitrary (NaN and inf scales included): they
    must reach neither the scores nor the mix."""
    B, Hq, Hkv, L, rK, rV = 3, 16, 4, 384, 48, 64
    lens = [300, 33, 0]
    q, P_K, P_V, kq, vq, ks, vs = _q8_case(7000, B, Hq, Hkv, L, rK, rV)
    kq, vq, ks, vs = kq.clone(), vq.clone(), ks.clone(), vs.clone()
    rng = np.random.default_rng(7001)
    bad = np.array([np.nan, np.inf, -np.inf, 3e38], np.float32)
    for b in range(B):
        n = L - lens[b]
        kq[b, :, lens[b]:] = torch.from_numpy(rng.integers(-128, 128, (Hkv, n, rK), dtype=np.int8))
        vq[b, :, lens[b]:] = torch.from_numpy(rng.integers(-128, 128, (Hkv, n, rV), dtype=np.int8))
        ks[b, :, lens[b]:] = torch.from_numpy(rng.choice(bad, (Hkv, n)))
        vs[b, :, lens[b]:] = torch.from_numpy(rng.choice(bad, (Hkv, n)))
    args = (q, P_K, P_V, kq, vq, ks, vs)
    got = _decode_q8(*args, lens, 384, num_splits)
    want = _oracle_q8(q, P_K, P_V, kq, vq, torch.nan_to_num(ks, 0.0, 0.0, 0.0),
                      torch.nan_to_num(vs, 0.0, 0.0, 0.0), lens)
    assert_decode_close(got, want)
    assert torch.all(got[2].float() == 0)


# ----------------------------------------------------------------------------- int8 page pools

def _q8_pools(B, Hkv, rK, rV, page_size, max_pages, spare, rng):
    num_pages = B * max_pages + spare
    table = rng.permutation(num_pages)[: B * max_pages].reshape(B, max_pages).astype(np.int32)
    kp = torch.full((num_pages, Hkv, page_size, rK), -128, dtype=torch.int8)
    vp = torch.full((num_pages, Hkv, page_size, rV), -128, dtype=torch.int8)
    ksp = torch.full((num_pages, Hkv, page_size), float("nan"), dtype=torch.float32)
    vsp = torch.full((num_pages, Hkv, page_size), float("nan"), dtype=torch.float32)
    return kp, vp, ksp, vsp, table


def _fill(pool, table, cache, page_size, upto):
    for b in range(table.shape[0]):
        for j in range(table.shape[1]):
            if j * page_size < upto[b]:
                pool[table[b, j]] = cache[b, :, j * page_size:(j + 1) * page_size]


def _decode_q8_paged(q, P_K, P_V, kp, vp, ksp, vsp, table, lens, max_seq_len, num_splits=0):
    B, Hq, d = q.shape
    out = torch.full((B, Hq, d), float("nan"), dtype=torch.bfloat16, device=DEV)
    ws = stief.workspace_for(B, Hq, P_K.shape[0], P_V.shape[2], max_seq_len)
    status = torch.zeros(1, dtype=torch.int32, device=DEV)
    stief.stief_decode_attention_q8_paged(q.to(DEV), P_K.to(DEV), P_V.to(DEV), kp.to(DEV), vp.to(DEV),
                                          ksp.to(DEV), vsp.to(DEV), torch.as_tensor(table).to(DEV),
                                          torch.as_tensor(np.asarray(lens, np.int32)).to(DEV), out, ws,
                                          max_seq_len, num_splits=num_splits, dev_status=status)
    assert stief.stief_read_device_status(status) == 0
    return out.cpu()


@pytest.mark.parametrize("page_size", [64, 128])
@pytest.mark.parametrize("num_splits", [0, 3])
def test_paged_q8_decode_matches_oracle(page_size, num_splits):
    """int8 codes and scales in shuffled page pools (NaN scales and -128 codes in every unused
    row): the decode over the pages equals the oracle's over the contiguous cache they stand
    for; block-table entries past each sequence's pages are -1."""
    rng = np.random.default_rng(8100 + page_size + num_splits)
    B, Hq, Hkv, rK, rV = 3, 16, 4, 64, 32
    max_pages = 1024 // page_size
    Lc = page_size * max_pages
    lens = [1000, 65, 0]
    q = si.queries(8100, B, Hq, 128)
    P_K, P_V = si.bases_bf16(8101, Hkv, 128, rK, rV)
    kq, ks = _random_q8_cache(8102, B, Hkv, Lc, rK)
    vq, vs = _random_q8_cache(8103, B, Hkv, Lc, rV)
    kp, vp, ksp, vsp, table = _q8_pools(B, Hkv, rK, rV, page_size, max_pages, 3, rng)
    for pool, cache in ((kp, kq), (vp, vq), (ksp, ks), (vsp, vs)):
        _fill(pool, table, cache, page_size, lens)
    for b in range(B):
        table[b, -(-lens[b] // page_size):] = -1
    got = _decode_q8_paged(q, P_K, P_V, kp, vp, ksp, vsp, table, lens, Lc, num_splits)
    want = oracle.decode(f64(q), f64(P_K), f64(P_V), oracle.dequantize_rows(kq.numpy(), ks.numpy()),
                         oracle.dequantize_rows(vq.numpy(), vs.numpy()), np.asarray(lens, np.int32))
    assert_decode_close(got, want)
    assert torch.all(got[2].float() == 0)


@pytest.mark.parametrize("T", [5, 200])
def test_paged_q8_compress_then_decode(T):
    """Compress chunks into int8 page pools (CUDA-core path for T < 128, tensor cores above),
    crossing pages, then decode over the pools; codes and scales equal the oracle's on the
    identity basis and the decode matches the oracle."""
    rng = np.random.default_rng(8200 + T)
    B, Hq, Hkv, rK, rV, page_size, max_pages = 2, 8, 2, 64, 64, 64, 8
    kp, vp, ksp, vsp, table = _q8_pools(B, Hkv, rK, rV, page_size, max_pages, 2, rng)
    # the rows below the starting lengths are attended to: valid codes and scales everywhere
    kp = torch.from_numpy(rng.integers(-127, 128, tuple(kp.shape), dtype=np.int8))
    vp = torch.from_numpy(rng.integers(-127, 128, tuple(vp.shape), dtype=np.int8))
    ksp = torch.from_numpy(rng.uniform(0.001, 0.02, tuple(ksp.shape)).astype(np.float32))
    vsp = torch.from_numpy(rng.uniform(0.001, 0.02, tuple(vsp.shape)).astype(np.float32))
    P_K, P_V = _identity_basis(Hkv, 128, rK), _identity_basis(Hkv, 128, rV)
    gk, gv, gks, gvs = kp.to(DEV), vp.to(DEV), ksp.to(DEV), vsp.to(DEV)
    gtab = torch.as_tensor(table).to(DEV)
    glens = torch.as_tensor(np.asarray([10, 50], np.int32)).to(DEV)
    k_new, v_new = si.full_kv(8200 + T, B, Hkv, T, 128)
    status = torch.zeros(1, dtype=torch.int32, device=DEV)
    stief.stief_compress_append_q8_paged(k_new.to(DEV), v_new.to(DEV), P_K.to(DEV), P_V.to(DEV), gk,
                                         gv, gks, gvs, gtab, glens, dev_status=status)
    assert stief.stief_read_device_status(status) == 0
    assert glens.cpu().tolist() == [10 + T, 50 + T]
    for b, L0 in enumerate([10, 50]):
        wk, wks = oracle.quantize_rows(f64(k_new[b])[..., :rK])
        for t in range(T):
            pg, row = table[b, (L0 + t) // page_size], (L0 + t) % page_size
            assert np.array_equal(gk[pg, :, row].cpu().numpy(), wk[:, t])
            assert np.array_equal(gks[pg, :, row].cpu().numpy(), wks[:, t])
    q = si.queries(8201, B, Hq, 128)
    lens = glens.cpu().tolist()
    got = _decode_q8_paged(q, P_K, P_V, gk.cpu(), gv.cpu(), gks.cpu(), gvs.cpu(), table, lens,
                           page_size * max_pages)
    Lc = page_size * max_pages
    kc = oracle.gather_pages(f64(gk.cpu()), table, lens, Lc)
    kcs = oracle.gather_pages(f64(gks.cpu())[..., None], table, lens, Lc)[..., 0]
    vc = oracle.gather_pages(f64(gv.cpu()), table, lens, Lc)
    vcs = oracle.gather_pages(f64(gvs.cpu())[..., None], table, lens, Lc)[..., 0]
    want = oracle.decode(f64(q), f64(P_K), f64(P_V), kc * kcs[..., None], vc * vcs[..., None],
                         np.asarray(lens, np.int32))
    assert_decode_close(got, want)


# ------------------------------------------------------------------------ the int8 fused step

def _append_decode_q8(q, k_new, v_new, P_K, P_V, kq, vq, ks, vs, lens, max_seq_len, num_splits=0,
                      expect_status=0):
    """One stief_append_decode_q8 call on device copies; returns (out, kq, vq, ks, vs, lens)."""
    B, Hq, d = q.shape
    dkq, dvq, dks, dvs = (x.to(DEV).contiguous() for x in (kq, vq, ks, vs))
    lens_t = torch.as_tensor(np.asarray(lens, np.int32)).to(DEV)
    out = torch.full((B, Hq, d), float("nan"), dtype=torch.bfloat16, device=DEV)
    ws = stief.workspace_for(B, Hq, P_K.shape[0], P_V.shape[2], max_seq_len)
    status = torch.zeros(1, dtype=torch.int32, device=DEV)
    stief.stief_append_decode_q8(q.to(DEV), k_new.to(DEV), v_new.to(DEV), P_K.to(DEV), P_V.to(DEV),
                                 dkq, dvq, dks, dvs, lens_t, out, ws, max_seq_len,
                                 num_splits=num_splits, dev_status=status)
    assert stief.stief_read_device_status(status) == expect_status
    return out.cpu(), dkq.cpu(), dvq.cpu(), dks.cpu(), dvs.cpu(), lens_t.cpu().numpy()


def _check_new_rows(kq0, vq0, ks0, vs0, gkq, gvq, gks, gvs, k_new, v_new, P_K, P_V, lens):
    """Row seq_lens[b] of every head holds the quantised projection of the new token (codes
    within one of the oracle's where the bf16 row may differ by an ulp, scales within a bf16
    ulp); every other row is unchanged."""
    B, Hkv = k_new.shape[:2]
    for b, L in enumerate(lens):
        for h in range(Hkv):
            for q0, s0, gq, gs, x, P in ((kq0, ks0, gkq, gks, k_new, P_K), (vq0, vs0, gvq, gvs, v_new, P_V)):
                lat = oracle.project(f64(x[b, h]).reshape(1, -1), f64(P[h]), round_to_bf16=True)
                wq, ws = oracle.quantize_rows(lat)
                got = gq[b, h, L].numpy().astype(np.int32)
                assert np.max(np.abs(got - wq[0].astype(np.int32))) <= 1
                np.testing.assert_allclose(gs[b, h, L].numpy(), ws[0], rtol=2 ** -7)
                keep = np.ones(q0.shape[2], bool)
                keep[L] = False
                assert torch.equal(gq[b, h][keep], q0[b, h][keep])
                assert torch.equal(gs[b, h][keep], s0[b, h][keep])


@pytest.mark.parametrize("rK,rV", [(64, 64), (32, 48), (96, 128)])
@pytest.mark.parametrize("num_splits", [0, 1, 3])
def test_append_decode_q8_matches_oracle(rK, rV, num_splits):
    """The int8 fused step: the new token's rows quantised into the cache at seq_lens[b]
    (as the compress stores them), the lengths incremented, and the output the oracle's decode
    over the grown cache (the stored codes and scales, dequantised)."""
    B, Hq, Hkv, L_max = 3, 16, 4, 768
    lens = [700, 33, 0]
    q, P_K, P_V, kq, vq, ks, vs = _q8_case(6900 + rK + num_splits, B, Hq, Hkv, L_max, rK, rV)
    k_new, v_new = si.full_kv(6950 + rV, B, Hkv, 1, 128)
    got, gkq, gvq, gks, gvs, glens = _append_decode_q8(q, k_new, v_new, P_K, P_V, kq, vq, ks, vs,
                                                       lens, 701, num_splits)
    assert glens.tolist() == [L + 1 for L in lens]
    _check_new_rows(kq, vq, ks, vs, gkq, gvq, gks, gvs, k_new[:, :, 0], v_new[:, :, 0], P_K, P_V, lens)
    want = _oracle_q8(q, P_K, P_V, gkq, gvq, gks, gvs, glens)
    assert_decode_close(got, want)


@pytest.mark.parametrize("Hq,Hkv", [(64, 8), (24, 4)])
def test_append_decode_q8_group_sizes(Hq, Hkv):
    """The int8 fused step with groups of 8 query heads per KV head (two MMA n-tiles) and of
    6 (two sub-groups of a KV head, only the first writes the cache row)."""
    B, L_max, rK, rV = 2, 512, 64, 48
    lens = [500, 77]
    q, P_K, P_V, kq, vq, ks, vs = _q8_case(7300 + Hq, B, Hq, Hkv, L_max, rK, rV)
    k_new, v_new = si.full_kv(7301 + Hq, B, Hkv, 1, 128)
    got, gkq, gvq, gks, gvs, glens = _append_decode_q8(q, k_new, v_new, P_K, P_V, kq, vq, ks, vs,
                                                       lens, 501)
    assert glens.tolist() == [L + 1 for L in lens]
    _check_new_rows(kq, vq, ks, vs, gkq, gvq, gks, gvs, k_new[:, :, 0], v_new[:, :, 0], P_K, P_V, lens)
    assert_decode_close(got, _oracle_q8(q, P_K, P_V, gkq, gvq, gks, gvs, glens))


def test_append_decode_q8_steps_follow_one_another():
    """Fused int8 steps back to back on one stream: each reads the row the previous one
    appended (the row just below its length, requested before its dependency wait and read
    again after it), and the final cache and output match the oracle."""
    B, Hq, Hkv, rK, rV, L_max = 2, 32, 8, 64, 64, 4096
    lens0 = [4000, 1500]
    q, P_K, P_V, kq, vq, ks, vs = _q8_case(7000, B, Hq, Hkv, L_max, rK, rV)
    dkq, dvq, dks, dvs = (x.to(DEV).contiguous() for x in (kq, vq, ks, vs))
    lens_t = torch.as_tensor(np.asarray(lens0, np.int32)).to(DEV)
    ws = stief.workspace_for(B, Hq, Hkv, rV, L_max)
    status = torch.zeros(1, dtype=torch.int32, device=DEV)
    gP_K, gP_V = P_K.to(DEV), P_V.to(DEV)
    steps = 5
    news = [si.full_kv(7001 + i, B, Hkv, 1, 128) for i in range(steps)]
    qs = [si.queries(7100 + i, B, Hq, 128).to(DEV) for i in range(steps)]
    outs = [torch.empty((B, Hq, 128), dtype=torch.bfloat16, device=DEV) for _ in range(steps)]
    for i in range(steps):
        stief.stief_append_decode_q8(qs[i], news[i][0].to(DEV), news[i][1].to(DEV), gP_K, gP_V,
                                     dkq, dvq, dks, dvs, lens_t, outs[i], ws, L_max,
                                     dev_status=status)
    assert stief.stief_read_device_status(status) == 0
    assert lens_t.cpu().tolist() == [L + steps for L in lens0]
    gkq, gvq, gks, gvs = dkq.cpu(), dvq.cpu(), dks.cpu(), dvs.cpu()
    for i in range(steps):
        step_lens = [L + i for L in lens0]
        # each step's rows, then the output over the cache as it stood after that step
        for b, L in enumerate(step_lens):
            for h in range(Hkv):
                for gq, gs, x, P in ((gkq, gks, news[i][0], P_K), (gvq, gvs, news[i][1], P_V)):
                    lat = oracle.project(f64(x[b, h, 0]).reshape(1, -1), f64(P[h]))
                    wq, wsc = oracle.quantize_rows(lat)
                    assert np.max(np.abs(gq[b, h, L].numpy().astype(np.int32) - wq[0])) <= 1
                    np.testing.assert_allclose(gs[b, h, L].numpy(), wsc[0], rtol=2 ** -7)
        want = _oracle_q8(qs[i].cpu(), P_K, P_V, gkq, gvq, gks, gvs, np.asarray(step_lens) + 1)
        assert_decode_close(outs[i].cpu(), want)
    # a plain int8 decode right after the last step on the same stream and caches
    for i in range(steps):
        stief.stief_append_decode_q8(qs[i], news[i][0].to(DEV), news[i][1].to(DEV), gP_K, gP_V,
                                     dkq, dvq, dks, dvs, lens_t, outs[i], ws, L_max,
                                     dev_status=status)
    out = torch.empty((B, Hq, 128), dtype=torch.bfloat16, device=DEV)
    stief.stief_decode_attention_q8(qs[0], gP_K, gP_V, dkq, dvq, dks, dvs, lens_t, out, ws, L_max,
                                    dev_status=status)
    assert stief.stief_read_device_status(status) == 0
    assert lens_t.cpu().tolist() == [L + 2 * steps for L in lens0]
    want = _oracle_q8(qs[0].cpu(), P_K, P_V, dkq.cpu(), dvq.cpu(), dks.cpu(), dvs.cpu(),
                      lens_t.cpu().numpy())
    assert_decode_close(out.cpu(), want)


def test_append_decode_q8_full_cache_is_refused():
    """A sequence whose cache is full is not appended to (capacity bit; its rows and length
    unchanged) and its output attends over the cache as it was; the other sequences step."""
    B, Hq, Hkv, rK, rV, L_max = 2, 16, 4, 64, 48, 256
    lens = [256, 100]
    q, P_K, P_V, kq, vq, ks, vs = _q8_case(7200, B, Hq, Hkv, L_max, rK, rV)
    k_new, v_new = si.full_kv(7201, B, Hkv, 1, 128)
    got, gkq, gvq, gks, gvs, glens = _append_decode_q8(
        q, k_new, v_new, P_K, P_V, kq, vq, ks, vs, lens, 256,
        expect_status=stief.DEV_CAPACITY_OVERFLOW)
    assert glens.tolist() == [256, 101]
    assert torch.equal(gkq[0], kq[0]) and torch.equal(gks[0], ks[0])
    want = _oracle_q8(q, P_K, P_V, gkq, gvq, gks, gvs, glens)
    assert_decode_close(got, want)
