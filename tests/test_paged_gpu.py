"""Paged latent caches: stief_decode_attention_paged, stief_compress_append_paged and
stief_append_decode_paged (CUDA, through the C ABI) against the fp64 oracle run on the
contiguous cache the pages stand for (oracle.gather_pages).

Pools are [num_pages][Hkv][page_size][r]; each sequence's pages are a random choice from the
pool (shuffled), and block-table entries past a sequence's pages hold -1 or ids of other
sequences' pages: only the pages below the length may be read.  Tolerance as for the
contiguous decode (2e-2 * ||o||_inf); compressed rows within the bound of the compress tests.
"""
import numpy as np
import pytest
import torch

import decode_attention_stief_b200 as stief
import oracle
import stief_inputs as si
from gpu_util import DECODE_TOL, assert_decode_close, decode_error, f64
from test_compress_gpu import _check_latent

pytestmark = pytest.mark.gpu
DEV = torch.device("cuda")


def _run_paged_decode(q, P_K, P_V, kpool, vpool, table, lens, max_seq_len, num_splits=0,
                      expect_status=0):
    B, Hq, d = q.shape
    out = torch.full((B, Hq, d), float("nan"), dtype=torch.bfloat16, device=DEV)
    ws = stief.workspace_for(B, Hq, P_K.shape[0], P_V.shape[2], max_seq_len)
    status = torch.zeros(1, dtype=torch.int32, device=DEV)
    stief.stief_decode_attention_paged(q.to(DEV), P_K.to(DEV), P_V.to(DEV), kpool.to(DEV),
                                       vpool.to(DEV), torch.as_tensor(table).to(DEV),
                                       torch.as_tensor(np.asarray(lens, np.int32)).to(DEV), out,
                                       ws, max_seq_len, num_splits=num_splits, dev_status=status)
    assert stief.stief_read_device_status(status) == expect_status
    return out.cpu()


def _fill_pages(pool, table, cache, page_size, upto):
    """Copy cache[b] rows of pages j * page_size < upto[b] into their pool pages."""
    for b in range(table.shape[0]):
        for j in range(table.shape[1]):
            if j * page_size < upto[b]:
                pool[table[b, j]] = cache[b, :, j * page_size:(j + 1) * page_size]


@pytest.mark.parametrize("page_size", [64, 128, 256])
@pytest.mark.parametrize("num_splits", [0, 1, 3])
def test_paged_decode_matches_contiguous(page_size, num_splits):
    rng = np.random.default_rng(page_size + num_splits)
    B, Hq, Hkv, rK, rV = 4, 16, 4, 64, 64
    max_pages = 1024 // page_size
    Lc = page_size * max_pages
    lens = [1000, 65, 0, 513]
    q = si.queries(5100, B, Hq, 128)
    P_K, P_V = si.bases_bf16(5100, Hkv, 128, rK, rV)
    kc = si.latent_cache(5100, B, Hkv, Lc, rK, 0)
    vc = si.latent_cache(5100, B, Hkv, Lc, rV, 1)
    kpool, vpool, table = _pools(B, Hkv, rK, rV, page_size, max_pages, 3, rng)
    _fill_pages(kpool, table, kc, page_size, [Lc] * B)
    _fill_pages(vpool, table, vc, page_size, [Lc] * B)
    got = _run_paged_decode(q, P_K, P_V, kpool, vpool, table, lens, max(lens), num_splits)
    want = oracle.decode(f64(q), f64(P_K), f64(P_V), oracle.gather_pages(f64(kpool), table, lens, Lc),
                         oracle.gather_pages(f64(vpool), table, lens, Lc), np.asarray(lens, np.int32))
    assert_decode_close(got, want)
    assert torch.all(got[2].float() == 0)


def _pools(B, Hkv, rK, rV, page_size, max_pages, spare, rng, fill=float("nan")):
    num_pages = B * max_pages + spare
    ids = rng.permutation(num_pages)[: B * max_pages].reshape(B, max_pages).astype(np.int32)
    kpool = torch.full((num_pages, Hkv, page_size, rK), fill, dtype=torch.bfloat16)
    vpool = torch.full((num_pages, Hkv, page_size, rV), fill, dtype=torch.bfloat16)
    return kpool, vpool, ids


@pytest.mark.parametrize("rK,rV", [(32, 48), (96, 64)])
def test_paged_decode_ranks_and_unmapped_tail(rK, rV):
    """Ranks with 64-token tiles (32/48) and 32-token tiles (96/64); block-table entries past
    each sequence's pages are -1 (never needed)."""
    rng = np.random.default_rng(rK)
    page_size, max_pages, B = 128, 6, 3
    lens = [700, 129, 256]
    q = si.queries(5200 + rK, B, 8, 128)
    P_K, P_V = si.bases_bf16(5200 + rK, 2, 128, rK, rV)
    kpool, vpool, table = _pools(B, 2, rK, rV, page_size, max_pages, 2, rng)
    kc = si.latent_cache(5201, B, 2, page_size * max_pages, rK, 0)
    vc = si.latent_cache(5201, B, 2, page_size * max_pages, rV, 1)
    _fill_pages(kpool, table, kc, page_size, lens)
    _fill_pages(vpool, table, vc, page_size, lens)
    for b in range(B):
        table[b, -(-lens[b] // page_size):] = -1  # pages past the length are not mapped
    got = _run_paged_decode(q, P_K, P_V, kpool, vpool, table, lens, page_size * max_pages)
    Lc = page_size * max_pages
    want = oracle.decode(f64(q), f64(P_K), f64(P_V), oracle.gather_pages(f64(kpool), table, lens, Lc),
                         oracle.gather_pages(f64(vpool), table, lens, Lc), np.asarray(lens, np.int32))
    assert_decode_close(got, want)


@pytest.mark.parametrize("T", [1, 7, 130, 300])
def test_paged_compress_append_crosses_pages(T):
    """Appends start mid-page and cross page boundaries (CUDA-core path for small T, tensor
    cores from 128 rows); rows land in the mapped pages, other rows stay untouched."""
    rng = np.random.default_rng(T)
    B, Hkv, rK, rV, page_size, max_pages = 2, 2, 64, 48, 64, 8
    lens0 = [60, 129]
    seed = 5300 + T
    k_new, v_new = si.full_kv(seed, B, Hkv, T, 128)
    P_K, P_V = si.bases_bf16(seed, Hkv, 128, rK, rV)
    kpool, vpool, table = _pools(B, Hkv, rK, rV, page_size, max_pages, 3, rng, fill=0.0)
    before_k, before_v = kpool.clone(), vpool.clone()
    lens_t = torch.as_tensor(np.asarray(lens0, np.int32)).to(DEV)
    gk, gv = kpool.to(DEV), vpool.to(DEV)
    status = torch.zeros(1, dtype=torch.int32, device=DEV)
    stief.stief_compress_append_paged(k_new.to(DEV), v_new.to(DEV), P_K.to(DEV), P_V.to(DEV), gk,
                                      gv, torch.as_tensor(table).to(DEV), lens_t, dev_status=status)
    assert stief.stief_read_device_status(status) == 0
    assert lens_t.cpu().tolist() == [L + T for L in lens0]
    gk, gv = gk.cpu(), gv.cpu()
    written = torch.zeros(kpool.shape[:3], dtype=torch.bool)
    for b, L in enumerate(lens0):
        rows_k = torch.stack([gk[table[b, t // page_size], :, t % page_size] for t in range(L, L + T)], 1)
        rows_v = torch.stack([gv[table[b, t // page_size], :, t % page_size] for t in range(L, L + T)], 1)
        for t in range(L, L + T):
            written[table[b, t // page_size], :, t % page_size] = True
        for h in range(Hkv):
            assert _check_latent(rows_k[h], f64(k_new[b, h]), f64(P_K[h])) > 0.98
            assert _check_latent(rows_v[h], f64(v_new[b, h]), f64(P_V[h])) > 0.98
    assert torch.equal(gk[~written], before_k[~written])
    assert torch.equal(gv[~written], before_v[~written])


def test_paged_compress_unmapped_page_is_reported():
    rng = np.random.default_rng(7)
    kpool, vpool, table = _pools(1, 2, 64, 64, 64, 4, 0, rng, fill=0.0)
    table[0, 2] = -1  # tokens 128..191 have no page
    k_new, v_new = si.full_kv(5400, 1, 2, 40, 128)
    P_K, P_V = si.bases_bf16(5400, 2, 128, 64, 64)
    status = torch.zeros(1, dtype=torch.int32, device=DEV)
    kpool, vpool = kpool.to(DEV), vpool.to(DEV)
    lens_after = torch.tensor([100], dtype=torch.int32, device=DEV)
    stief.stief_compress_append_paged(k_new.to(DEV), v_new.to(DEV), P_K.to(DEV), P_V.to(DEV),
                                      kpool, vpool, torch.as_tensor(table).to(DEV), lens_after,
                                      dev_status=status)
    assert stief.stief_read_device_status(status) & stief.DEV_CAPACITY_OVERFLOW
    # all or nothing: no row written, the length unchanged
    assert torch.all(kpool.to(DEV) == 0) and lens_after.item() == 100


def test_paged_append_decode_steps():
    """Three fused steps over a paged cache equal three oracle steps on the contiguous cache;
    the new token's page may be a fresh one (its first row)."""
    rng = np.random.default_rng(11)
    B, Hq, Hkv, rK, rV, page_size, max_pages = 3, 16, 4, 64, 64, 64, 6
    lens = [127, 64, 0]  # the first steps write rows 127 (end of a page), 64 and 0 (page starts)
    Lc = page_size * max_pages
    q = si.queries(5500, B, Hq, 128)
    P_K, P_V = si.bases_bf16(5500, Hkv, 128, rK, rV)
    kpool, vpool, table = _pools(B, Hkv, rK, rV, page_size, max_pages, 2, rng, fill=0.0)
    kc = si.latent_cache(5501, B, Hkv, Lc, rK, 0)
    vc = si.latent_cache(5501, B, Hkv, Lc, rV, 1)
    _fill_pages(kpool, table, kc, page_size, lens)
    _fill_pages(vpool, table, vc, page_size, lens)
    gk, gv, gt = kpool.to(DEV), vpool.to(DEV), torch.as_tensor(table).to(DEV)
    lens_t = torch.as_tensor(np.asarray(lens, np.int32)).to(DEV)
    ws = stief.workspace_for(B, Hq, Hkv, rV, Lc)
    wk = oracle.gather_pages(f64(kpool), table, lens, Lc)
    wv = oracle.gather_pages(f64(vpool), table, lens, Lc)
    wl = np.asarray(lens, np.int32)
    for step in range(3):
        kn, vn = si.full_kv(5600 + step, B, Hkv, 1, 128)
        out = torch.full((B, Hq, 128), float("nan"), dtype=torch.bfloat16, device=DEV)
        status = torch.zeros(1, dtype=torch.int32, device=DEV)
        stief.stief_append_decode_paged(q.to(DEV), kn.to(DEV), vn.to(DEV), P_K.to(DEV), P_V.to(DEV),
                                        gk, gv, gt, lens_t, out, ws, Lc, dev_status=status)
        assert stief.stief_read_device_status(status) == 0
        wk, wv, wl, _ = oracle.compress_append(f64(kn), f64(vn), f64(P_K), f64(P_V), wk, wv, wl)
        want = oracle.decode(f64(q), f64(P_K), f64(P_V), wk, wv, wl)
        assert lens_t.cpu().tolist() == wl.tolist()
        err = decode_error(out.cpu(), want)
        assert err <= DECODE_TOL, err
        assert int(ws[:256].count_nonzero()) == 0


def test_paged_append_into_unmapped_page_is_refused():
    rng = np.random.default_rng(12)
    kpool, vpool, table = _pools(1, 2, 64, 64, 64, 4, 0, rng, fill=0.0)
    table[0, 1] = -1  # token 64 has no page
    q = si.queries(5700, 1, 8, 128)
    P_K, P_V = si.bases_bf16(5700, 2, 128, 64, 64)
    kn, vn = si.full_kv(5701, 1, 2, 1, 128)
    lens_t = torch.tensor([64], dtype=torch.int32, device=DEV)
    out = torch.empty((1, 8, 128), dtype=torch.bfloat16, device=DEV)
    status = torch.zeros(1, dtype=torch.int32, device=DEV)
    stief.stief_append_decode_paged(q.to(DEV), kn.to(DEV), vn.to(DEV), P_K.to(DEV), P_V.to(DEV),
                                    kpool.to(DEV), vpool.to(DEV), torch.as_tensor(table).to(DEV),
                                    lens_t, out, stief.workspace_for(1, 8, 2, 64, 256), 256,
                                    dev_status=status)
    assert stief.stief_read_device_status(status) & stief.DEV_CAPACITY_OVERFLOW
    assert lens_t.item() == 64


def test_paged_decode_multi_wave_grid():
    """More units than SMs (40 x 8 = 320): the paged decode in the two-CTAs-per-SM plan."""
    rng = np.random.default_rng(13)
    B, Hq, Hkv, rK, rV, page_size, max_pages = 40, 32, 8, 64, 64, 64, 5
    Lc = page_size * max_pages
    lens = rng.integers(1, Lc, size=B).tolist()
    lens[2] = 0
    q = si.queries(5800, B, Hq, 128)
    P_K, P_V = si.bases_bf16(5800, Hkv, 128, rK, rV)
    kpool, vpool, table = _pools(B, Hkv, rK, rV, page_size, max_pages, 4, rng)
    kc = si.latent_cache(5801, B, Hkv, Lc, rK, 0)
    vc = si.latent_cache(5801, B, Hkv, Lc, rV, 1)
    _fill_pages(kpool, table, kc, page_size, [Lc] * B)
    _fill_pages(vpool, table, vc, page_size, [Lc] * B)
    got = _run_paged_decode(q, P_K, P_V, kpool, vpool, table, lens, Lc)
    want = oracle.decode(f64(q), f64(P_K), f64(P_V), oracle.gather_pages(f64(kpool), table, lens, Lc),
                         oracle.gather_pages(f64(vpool), table, lens, Lc), np.asarray(lens, np.int32))
    assert_decode_close(got, want)
