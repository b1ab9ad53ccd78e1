"""Compress/append parity: stief_compress_append (CUDA, through the C ABI) against the oracle.

The latent is the bf16 RNE of an fp32-accumulated product, so it must lie within
half a bf16 ulp plus the fp32 dot-product error bound (gamma_128 * sum |x_i p_i|)
of the exact product, and at least 98% of elements must equal the oracle's RNE of
the exact product bit for bit (they differ only where the exact value sits within
the fp32 error of a rounding boundary, or where the result nearly cancels).
Cache indexing and lengths must be bit-exact.
"""
import numpy as np
import pytest
import torch

import decode_attention_stief_b200 as stief
import oracle
import stief_inputs as si
from gpu_util import (assert_decode_close, bf16_ulp, f64, gpu_decode, oracle_decode)

pytestmark = pytest.mark.gpu

CANARY_K = 0x7FC1  # a quiet-NaN bf16 pattern: any stray write changes it
CANARY_V = 0xFFC3


def _s16(pattern: int) -> int:
    """A 16-bit pattern as the signed int16 value with the same bits."""
    return int(np.uint16(pattern).view(np.int16))


def _cache(B, Hkv, L_max, r, pattern):
    return torch.full((B, Hkv, L_max, r), _s16(pattern), dtype=torch.int16).view(torch.bfloat16)


def _run_append(k_new, v_new, P_K, P_V, k_lat, v_lat, lens, expect_status=0):
    dev = torch.device("cuda")
    args = [x.to(dev).contiguous() for x in (k_new, v_new, P_K, P_V, k_lat, v_lat)]
    lens_t = torch.as_tensor(np.asarray(lens, np.int32)).to(dev)
    status = torch.zeros(1, dtype=torch.int32, device=dev)
    stief.stief_compress_append(*args, lens_t, dev_status=status)
    st = stief.stief_read_device_status(status)
    assert st == expect_status, f"device status {st:#x}"
    return args[4].cpu(), args[5].cpu(), lens_t.cpu().numpy()


# forward error bound of a d-term dot product accumulated in fp32 (any order):
# |fl(x.p) - x.p| <= gamma_d * sum_i |x_i p_i|, gamma_d = d u / (1 - d u), u = 2^-24
GAMMA_128 = 128 * 2.0 ** -24 / (1 - 128 * 2.0 ** -24)


def _check_latent(got_bits: torch.Tensor, x: np.ndarray, P: np.ndarray):
    """got = RNE_bf16(fp32 accumulation of x . P): within half a bf16 ulp of the fp32 value,
    which is within gamma_128 * sum|x_i p_i| of the exact product.  Returns the fraction of
    elements equal to the oracle's RNE of the exact product."""
    g = f64(got_bits)
    exact = oracle.project(x, P, round_to_bf16=False)
    want = oracle.project(x, P, round_to_bf16=True)
    bound = 0.5 * bf16_ulp(np.maximum(np.abs(g), np.abs(exact))) + \
        GAMMA_128 * (np.abs(x) @ np.abs(P))
    err = np.abs(g - exact)
    assert np.all(err <= bound), f"max excess {np.max(err - bound)}"
    return float(np.mean(g == want))


@pytest.mark.parametrize("T", [1, 3, 8, 9, 40, 200])
@pytest.mark.parametrize("rK,rV", [(64, 64), (32, 48), (16, 128), (96, 112)])
def test_append_matches_oracle(T, rK, rV):
    B, Hkv, d, L_max = 2, 3, 128, 260
    seed = 10 * T + rK
    k_new, v_new = si.full_kv(seed, B, Hkv, T, d)
    P_K, P_V = si.bases_bf16(seed, Hkv, d, rK, rV)
    lens = [5, 60]
    k_lat = _cache(B, Hkv, L_max, rK, CANARY_K)
    v_lat = _cache(B, Hkv, L_max, rV, CANARY_V)
    gk, gv, glens = _run_append(k_new, v_new, P_K, P_V, k_lat, v_lat, lens)
    assert glens.tolist() == [L + T for L in lens]
    for b, L in enumerate(lens):
        for h in range(Hkv):
            exact_k = _check_latent(gk[b, h, L:L + T], f64(k_new[b, h]), f64(P_K[h]))
            exact_v = _check_latent(gv[b, h, L:L + T], f64(v_new[b, h]), f64(P_V[h]))
            assert exact_k > 0.98 and exact_v > 0.98
            keep = np.ones(L_max, bool)
            keep[L:L + T] = False
            assert torch.all(gk[b, h, keep].view(torch.int16) == _s16(CANARY_K))
            assert torch.all(gv[b, h, keep].view(torch.int16) == _s16(CANARY_V))


def test_identity_basis_is_bit_exact():
    B, Hkv, T, d, r, L_max = 1, 2, 37, 128, 48, 64
    k_new, v_new = si.full_kv(3, B, Hkv, T, d)
    P = torch.zeros((Hkv, d, r))
    P[:, torch.arange(r), torch.arange(r)] = 1.0
    P = P.to(torch.bfloat16)
    gk, gv, _ = _run_append(k_new, v_new, P, P, _cache(B, Hkv, L_max, r, 0),
                            _cache(B, Hkv, L_max, r, 0), [0])
    assert torch.equal(gk[:, :, :T], k_new[..., :r])
    assert torch.equal(gv[:, :, :T], v_new[..., :r])


def test_capacity_overflow_leaves_sequence_untouched():
    B, Hkv, T, d, r, L_max = 3, 2, 3, 128, 32, 10
    k_new, v_new = si.full_kv(4, B, Hkv, T, d)
    P_K, P_V = si.bases_bf16(4, Hkv, d, r, r)
    lens = [0, 7, 8]                 # the second fits exactly, the third overflows
    k_lat = _cache(B, Hkv, L_max, r, CANARY_K)
    v_lat = _cache(B, Hkv, L_max, r, CANARY_K)
    gk, gv, glens = _run_append(k_new, v_new, P_K, P_V, k_lat, v_lat, lens,
                                expect_status=stief.DEV_CAPACITY_OVERFLOW)
    assert glens.tolist() == [3, 10, 8]
    assert torch.all(gk[2].view(torch.int16) == _s16(CANARY_K))
    assert torch.all(gv[2].view(torch.int16) == _s16(CANARY_K))
    _, _, olens, nbad = oracle.compress_append(f64(k_new), f64(v_new), f64(P_K), f64(P_V),
                                               f64(k_lat), f64(v_lat), lens)
    assert nbad == 1 and olens.tolist() == glens.tolist()


def test_negative_length_is_reported():
    B, Hkv, T, d, r, L_max = 2, 1, 2, 128, 16, 8
    k_new, v_new = si.full_kv(5, B, Hkv, T, d)
    P_K, P_V = si.bases_bf16(5, Hkv, d, r, r)
    gk, gv, glens = _run_append(k_new, v_new, P_K, P_V, _cache(B, Hkv, L_max, r, CANARY_K),
                                _cache(B, Hkv, L_max, r, CANARY_K), [-1, 0],
                                expect_status=stief.DEV_BAD_LENGTH)
    assert glens.tolist() == [-1, 2]
    assert torch.all(gk[0].view(torch.int16) == _s16(CANARY_K))


def test_append_then_decode_end_to_end():
    """Prefill chunk + single-token appends, then decode; each side compresses itself."""
    B, Hq, Hkv, d, rK, rV, L_max = 2, 8, 2, 128, 64, 48, 600
    seed = 77
    P_K, P_V = si.bases_bf16(seed, Hkv, d, rK, rV)
    k_lat = torch.zeros((B, Hkv, L_max, rK), dtype=torch.bfloat16)
    v_lat = torch.zeros((B, Hkv, L_max, rV), dtype=torch.bfloat16)
    ok_lat, ov_lat = f64(k_lat), f64(v_lat)
    lens = np.zeros(B, np.int32)
    olens = lens.copy()
    dev = torch.device("cuda")
    gk, gv = k_lat.to(dev), v_lat.to(dev)
    glens = torch.as_tensor(lens).to(dev)
    for step, T in enumerate([500, 1, 1, 1, 7]):
        k_new, v_new = si.full_kv(seed + step, B, Hkv, T, d)
        stief.stief_compress_append(k_new.to(dev), v_new.to(dev), P_K.to(dev), P_V.to(dev),
                                    gk, gv, glens)
        ok_lat, ov_lat, olens, nbad = oracle.compress_append(
            f64(k_new), f64(v_new), f64(P_K), f64(P_V), ok_lat, ov_lat, olens)
        assert nbad == 0
    torch.cuda.synchronize()
    assert glens.cpu().numpy().tolist() == olens.tolist() == [510, 510]
    q = si.queries(seed, B, Hq, d)
    got = gpu_decode(q, P_K, P_V, gk, gv, olens)
    want = oracle.decode(f64(q), f64(P_K), f64(P_V), ok_lat, ov_lat, olens)
    assert_decode_close(got, want)


@pytest.mark.parametrize("T,rK,rV", [(128, 64, 64), (300, 32, 48), (257, 96, 112), (640, 16, 128)])
def test_tensor_core_chunks(T, rK, rV):
    """Prefill-sized appends (T >= 128) run on the tcgen05 path: full tiles and ragged tails."""
    B, Hkv, d, L_max = 2, 2, 128, T + 40
    seed = 1000 + T + rK
    k_new, v_new = si.full_kv(seed, B, Hkv, T, d)
    P_K, P_V = si.bases_bf16(seed, Hkv, d, rK, rV)
    lens = [0, 33]
    gk, gv, glens = _run_append(k_new, v_new, P_K, P_V, _cache(B, Hkv, L_max, rK, CANARY_K),
                                _cache(B, Hkv, L_max, rV, CANARY_V), lens)
    assert glens.tolist() == [L + T for L in lens]
    for b, L in enumerate(lens):
        for h in range(Hkv):
            assert _check_latent(gk[b, h, L:L + T], f64(k_new[b, h]), f64(P_K[h])) > 0.98
            assert _check_latent(gv[b, h, L:L + T], f64(v_new[b, h]), f64(P_V[h])) > 0.98
            keep = np.ones(L_max, bool)
            keep[L:L + T] = False
            assert torch.all(gk[b, h, keep].view(torch.int16) == _s16(CANARY_K))
            assert torch.all(gv[b, h, keep].view(torch.int16) == _s16(CANARY_V))


def test_prefill_chunk_full_size():
    """One layer of the prefill workload: a 4096-token chunk for 8 KV heads, ranks 64/64."""
    w = si.PREFILL_CHUNK
    B, Hkv, T, d, rK, rV = w["B"], w["Hkv"], w["T"], w["d"], w["rK"], w["rV"]
    dev = torch.device("cuda")
    k_new = si.low_rank_rows_torch(si.sub_seed(w["seed"], 1), B * Hkv, T, d, dev).view(B, Hkv, T, d)
    v_new = si.low_rank_rows_torch(si.sub_seed(w["seed"], 2), B * Hkv, T, d, dev).view(B, Hkv, T, d)
    P_K, P_V = si.bases_bf16(w["seed"], Hkv, d, rK, rV)
    gk, gv, glens = _run_append(k_new, v_new, P_K, P_V,
                                torch.zeros((B, Hkv, T, rK), dtype=torch.bfloat16),
                                torch.zeros((B, Hkv, T, rV), dtype=torch.bfloat16), [0])
    assert glens.tolist() == [T]
    for h in range(Hkv):
        assert _check_latent(gk[0, h], f64(k_new[0, h]), f64(P_K[h])) > 0.98
        assert _check_latent(gv[0, h], f64(v_new[0, h]), f64(P_V[h])) > 0.98


@pytest.mark.parametrize("rK,rV", [(64, 64), (32, 48)])
def test_decode_right_after_compress_same_stream(rK, rV):
    """Compress chunks (tensor-core and CUDA-core paths) and decodes issued back to back on one
    stream with no host synchronisation and no other work in between.  The compress call's
    length kernel lets the next kernel start early, so the decode that follows must request no
    cache row before its dependency wait: the caches start as NaN, so a row read before the
    compress wrote it would show in the output."""
    B, Hq, Hkv, d, L_max = 2, 16, 4, 128, 2048
    seed = 91
    dev = torch.device("cuda")
    chunks = [640, 300, 1, 128, 7, 900]
    P_K, P_V = si.bases_bf16(seed, Hkv, d, rK, rV)
    gPK, gPV = P_K.to(dev), P_V.to(dev)
    gk = torch.full((B, Hkv, L_max, rK), float("nan"), dtype=torch.bfloat16, device=dev)
    gv = torch.full((B, Hkv, L_max, rV), float("nan"), dtype=torch.bfloat16, device=dev)
    glens = torch.zeros(B, dtype=torch.int32, device=dev)
    news = [si.full_kv(seed + i, B, Hkv, T, d) for i, T in enumerate(chunks)]
    gnews = [(k.to(dev), v.to(dev)) for k, v in news]
    qs = [si.queries(seed + 50 + i, B, Hq, d) for i in range(len(chunks))]
    gqs = [q.to(dev) for q in qs]
    outs = [torch.empty((B, Hq, d), dtype=torch.bfloat16, device=dev) for _ in chunks]
    max_seq = sum(chunks)
    ws = stief.workspace_for(B, Hq, Hkv, rV, max_seq)
    status = torch.zeros(1, dtype=torch.int32, device=dev)
    torch.cuda.synchronize()
    for i in range(len(chunks)):
        stief.stief_compress_append(gnews[i][0], gnews[i][1], gPK, gPV, gk, gv, glens,
                                    dev_status=status)
        stief.stief_decode_attention(gqs[i], gPK, gPV, gk, gv, glens, outs[i], ws, max_seq,
                                     dev_status=status)
    assert stief.stief_read_device_status(status) == 0
    ok_lat = np.zeros((B, Hkv, L_max, rK))
    ov_lat = np.zeros((B, Hkv, L_max, rV))
    olens = np.zeros(B, np.int32)
    for i in range(len(chunks)):
        ok_lat, ov_lat, olens, nbad = oracle.compress_append(
            f64(news[i][0]), f64(news[i][1]), f64(P_K), f64(P_V), ok_lat, ov_lat, olens)
        assert nbad == 0
        want = oracle.decode(f64(qs[i]), f64(P_K), f64(P_V), ok_lat, ov_lat, olens)
        assert_decode_close(outs[i].cpu(), want)
    assert glens.cpu().numpy().tolist() == olens.tolist() == [max_seq] * B


@pytest.mark.parametrize("name", ["llama3_8b_32k", "llama31_8b_128k"])
def test_compress_then_decode_full_size(name):
    """A benchmark shape built the way the model would build it: the whole context compressed by
    one stief_compress_append call (tensor-core path), then a decode over that cache; the
    stored latents are checked against the exact products and the decode against the oracle's
    decode over the oracle's own compressed cache."""
    w = si.WORKLOADS[name]
    B, Hq, Hkv, d, L, rK, rV = w.B, w.Hq, w.Hkv, w.d, w.L, w.rK, w.rV
    dev = torch.device("cuda")
    seed = si.sub_seed(w.seed, 61)
    k_new = si.low_rank_rows_torch(si.sub_seed(seed, 1), B * Hkv, L, d, dev).view(B, Hkv, L, d)
    v_new = si.low_rank_rows_torch(si.sub_seed(seed, 2), B * Hkv, L, d, dev).view(B, Hkv, L, d)
    P_K, P_V = si.bases_bf16(seed, Hkv, d, rK, rV)
    gk, gv, glens = _run_append(k_new, v_new, P_K, P_V,
                                torch.zeros((B, Hkv, L, rK), dtype=torch.bfloat16),
                                torch.zeros((B, Hkv, L, rV), dtype=torch.bfloat16), [0] * B)
    assert glens.tolist() == [L] * B
    kn, vn = f64(k_new.cpu()), f64(v_new.cpu())
    for h in (0, Hkv - 1):  # two heads checked element by element (the decode covers all)
        assert _check_latent(gk[0, h], kn[0, h], f64(P_K[h])) > 0.98
        assert _check_latent(gv[0, h], vn[0, h], f64(P_V[h])) > 0.98
    q = si.queries_torch(seed + 3, B, Hq, d, dev)
    got = gpu_decode(q, P_K, P_V, gk, gv, [L] * B)
    ok_lat, ov_lat, olens, nbad = oracle.compress_append(
        kn, vn, f64(P_K), f64(P_V), np.zeros((B, Hkv, L, rK)), np.zeros((B, Hkv, L, rV)),
        np.zeros(B, np.int32))
    assert nbad == 0 and olens.tolist() == [L] * B
    want = oracle.decode(f64(q.cpu()), f64(P_K), f64(P_V), ok_lat, ov_lat, olens)
    assert_decode_close(got, want)
