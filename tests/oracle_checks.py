"""Pins for the fp64 oracle, written as functions of an ``oracle.Oracle`` object.

Each check ties the oracle to something other than itself: a library routine
(torch's float32->bfloat16 conversion, torch's scaled_dot_product_attention in
float64), a closed form, an invariance the pages state, or exact arithmetic.
``test_oracle_pins.py`` runs them on the oracle; ``test_oracle_mutants.py`` runs
them on copies of the oracle with a planted mistake and expects a failure.

Pages: "Don't be so Stief! Learning KV Cache low-rank approximation over the
Stiefel manifold", StiefAttention technical summary, "Mecanismo Central" /
"Kernmechanismus": item 2 (orthonormal bases on the Stiefel manifold), item 3
(QR orthonormalisation; R is only a change of coordinates inside the subspace),
item 5 (stored K_down = K P_K, reconstruction K~ = K_down P_K^T before
attention; the bases may be folded into the attention weights); "Resultados Experimentais"
(the uncompressed FP16 baseline, i.e. plain attention, which the r = d case must reproduce).
STAR-KV technical summary, "Metodologia" item 2 (values decomposed jointly over the heads,
keys per head) for the joint-value calls.
"""
from __future__ import annotations

import math

import numpy as np
import torch
import torch.nn.functional as F

import stief_inputs as si


def _rel_err(a: np.ndarray, b: np.ndarray) -> float:
    scale = max(float(np.max(np.abs(b))), 1e-300)
    return float(np.max(np.abs(a - b))) / scale


def _identity_basis(d: int, r: int) -> np.ndarray:
    """P = [I_r; 0]: the first r columns of the d x d identity (exactly representable)."""
    P = np.zeros((d, r))
    P[np.arange(r), np.arange(r)] = 1.0
    return P


# ----------------------------------------------------------------------------- bf16 rounding

def check_round_bf16_matches_torch(o, n: int = 200_000, seed: int = 0) -> None:
    """RNE to bf16 equals torch's float32 -> bfloat16 conversion on float32 inputs."""
    rng = np.random.default_rng(seed)
    mant = rng.uniform(1.0, 2.0, n)
    expo = rng.integers(-140, 128, n)
    sign = np.where(rng.random(n) < 0.5, -1.0, 1.0)
    x32 = (sign * mant * np.exp2(expo.astype(np.float64))).astype(np.float32)
    # also every tie pattern: low 16 bits exactly 0x8000 around random high halves
    hi = rng.integers(0, 0x7F7F, 4096, dtype=np.uint32)
    ties = ((hi << 16) | 0x8000).astype(np.uint32).view(np.float32)
    x32 = np.concatenate([x32, ties, -ties])
    ref = torch.from_numpy(x32).to(torch.bfloat16).to(torch.float64).numpy()
    got = o.round_bf16(x32.astype(np.float64))
    assert np.array_equal(got, ref), "bf16 rounding differs from torch's float32->bf16"


def check_round_bf16_edges(o) -> None:
    """Hand-derived cases: ties to even, subnormal grid, overflow to infinity."""
    cases = [
        (1.0 + 2.0 ** -8, 1.0),                       # tie, 1.0 has an even last bit
        (1.0 + 3 * 2.0 ** -8, 1.0 + 2.0 ** -6),       # tie, rounds up to the even neighbour
        (1.0 + 2.0 ** -8 + 2.0 ** -30, 1.0 + 2.0 ** -7),  # just above the tie
        (-(1.0 + 2.0 ** -8), -1.0),
        (2.0 ** -133, 2.0 ** -133),                   # smallest subnormal
        (2.0 ** -134, 0.0),                           # tie between 0 and 2^-133 -> 0
        (3 * 2.0 ** -134, 2.0 ** -132),               # tie between 1 and 2 ulps -> 2
        ((2 - 2.0 ** -7) * 2.0 ** 127, (2 - 2.0 ** -7) * 2.0 ** 127),  # largest finite
        ((2 - 2.0 ** -8) * 2.0 ** 127, math.inf),     # tie above the largest -> overflow
        (0.0, 0.0),
    ]
    x = np.array([c[0] for c in cases])
    want = np.array([c[1] for c in cases])
    got = o.round_bf16(x)
    assert np.array_equal(got, want), f"bf16 edge cases: got {got}, want {want}"


# ----------------------------------------------------------------------------- bases

def check_qr_bases_orthonormal(d: int = 128, ranks=(16, 32, 48, 64, 96, 128)) -> None:
    """P^T P = I to 1e-6 for the QR-generated bases (before bf16 rounding)."""
    for r in ranks:
        P = si.bases(1234, 2, d, r)
        for h in range(P.shape[0]):
            err = np.max(np.abs(P[h].T @ P[h] - np.eye(r)))
            assert err <= 1e-6, f"P^T P - I = {err} for r={r}"


# ----------------------------------------------------------------------------- attention

def _sdpa_reference(q, K, V, lens) -> np.ndarray:
    """Textbook softmax attention (torch SDPA, float64, GQA by contiguous groups)."""
    B, Hq, d = q.shape
    out = np.zeros_like(q)
    for b in range(B):
        L = int(lens[b])
        if L == 0:
            continue
        qt = torch.from_numpy(q[b][None, :, None, :])          # [1, Hq, 1, d]
        kt = torch.from_numpy(np.ascontiguousarray(K[b][None, :, :L, :]))
        vt = torch.from_numpy(np.ascontiguousarray(V[b][None, :, :L, :]))
        o = F.scaled_dot_product_attention(qt, kt, vt, enable_gqa=True)
        out[b] = o[0, :, 0, :].numpy()
    return out


def check_full_rank_is_plain_attention(o, q_scale: float = 1.0, d: int = 128,
                                       tol: float = 1e-12) -> None:
    """r = d: P is square orthogonal, so the method is exactly uncompressed attention."""
    B, Hq, Hkv, L_max = 2, 8, 2, 40
    lens = np.array([37, 5], dtype=np.int32)
    rng = np.random.default_rng(11)
    K = np.stack([si.low_rank_rows(rng, L_max, d) for _ in range(B * Hkv)]).reshape(B, Hkv, L_max, d)
    V = np.stack([si.low_rank_rows(rng, L_max, d) for _ in range(B * Hkv)]).reshape(B, Hkv, L_max, d)
    q = q_scale * rng.standard_normal((B, Hq, d))
    P_K = si.bases(21, Hkv, d, d)
    P_V = si.bases(22, Hkv, d, d)
    zk = np.zeros((B, Hkv, L_max, d))
    k_lat, v_lat, _, nbad = o.compress_append(K, V, P_K, P_V, zk, zk.copy(),
                                              np.zeros(B, np.int32), round_to_bf16=False)
    assert nbad == 0
    got = o.decode(q, P_K, P_V, k_lat, v_lat, lens)
    want = _sdpa_reference(q, K, V, lens)
    assert np.all(np.isfinite(got)), "non-finite output"
    err = _rel_err(got, want)
    assert err <= tol, f"r=d differs from plain attention: rel err {err}"


def check_tiny_compressed_is_sdpa_on_reconstructed_rows(o) -> None:
    """Brute force on tiny inputs with r < d (d = 16, r_K = 8, r_V = 4, up to 5 tokens): the
    rows K~ = K_down P_K^T and V~ = V_down P_V^T formed explicitly (numpy products), then torch
    SDPA in float64 over them, must equal the oracle's decode to 1e-13."""
    d, rK, rV, B, Hq, Hkv, L_max = 16, 8, 4, 3, 4, 2, 5
    rng = np.random.default_rng(40)
    lens = np.array([5, 1, 3], np.int32)
    P_K = si.bases(41, Hkv, d, rK)
    P_V = si.bases(42, Hkv, d, rV)
    k = rng.standard_normal((B, Hkv, L_max, rK))
    v = rng.standard_normal((B, Hkv, L_max, rV))
    q = rng.standard_normal((B, Hq, d))
    K = np.einsum("bhtr,hdr->bhtd", k, P_K)
    V = np.einsum("bhtr,hdr->bhtd", v, P_V)
    want = _sdpa_reference(q, K, V, lens)
    got = o.decode(q, P_K, P_V, k, v, lens)
    assert _rel_err(got, want) <= 1e-13


def check_gauge_invariance(o, r: int = 48, d: int = 128) -> None:
    """P -> P.O (O orthogonal r x r) leaves the output unchanged (QR: R is a change of coordinates)."""
    B, Hq, Hkv, L = 2, 4, 2, 29
    rng = np.random.default_rng(12)
    K = np.stack([si.low_rank_rows(rng, L, d) for _ in range(B * Hkv)]).reshape(B, Hkv, L, d)
    V = np.stack([si.low_rank_rows(rng, L, d) for _ in range(B * Hkv)]).reshape(B, Hkv, L, d)
    q = rng.standard_normal((B, Hq, d))
    lens = np.array([L, 17], dtype=np.int32)
    P_K = si.bases(31, Hkv, d, r)
    P_V = si.bases(32, Hkv, d, r)
    O = np.stack([si.stiefel_basis(rng, r, r) for _ in range(Hkv)])
    outs = []
    for PK, PV in ((P_K, P_V), (P_K @ O, P_V @ O)):
        z = np.zeros((B, Hkv, L, r))
        kl, vl, _, _ = o.compress_append(K, V, PK, PV, z, z.copy(), np.zeros(B, np.int32),
                                         round_to_bf16=False)
        outs.append(o.decode(q, PK, PV, kl, vl, lens))
    err = _rel_err(outs[1], outs[0])
    assert err <= 1e-12, f"basis change moved the output: rel err {err}"


def check_single_token(o, r: int = 64, d: int = 128) -> None:
    """L = 1: softmax of one score is 1, so o = V~_0 whatever q and K are."""
    rng = np.random.default_rng(13)
    B, Hq, Hkv = 1, 4, 1
    P_K = si.bases(41, Hkv, d, r)
    P_V = _identity_basis(d, r)[None]
    k_lat = rng.standard_normal((B, Hkv, 3, r))
    v_lat = rng.standard_normal((B, Hkv, 3, r))
    q = 5.0 * rng.standard_normal((B, Hq, d))
    got = o.decode(q, P_K, P_V, k_lat, v_lat, np.array([1], np.int32))
    want = np.zeros((B, Hq, d))
    want[:, :, :r] = v_lat[0, 0, 0]
    assert np.array_equal(got, want), "one-token output is not the reconstructed value row"


def check_two_tokens(o, r: int = 64, d: int = 128) -> None:
    """Two tokens with scores a/sqrt(d) and 0: weights sigma(a/sqrt(d)) and 1 - sigma."""
    Hq = 4
    a = np.array([0.5, 3.0, -7.0, 20.0])
    P = _identity_basis(d, r)[None]
    q = np.zeros((1, Hq, d))
    q[0, :, 0] = a
    k_lat = np.zeros((1, 1, 2, r))
    k_lat[0, 0, 0, 0] = 1.0
    v_lat = np.zeros((1, 1, 2, r))
    v_lat[0, 0, 0, 1] = 1.0
    v_lat[0, 0, 1, 2] = 1.0
    got = o.decode(q, P, P, k_lat, v_lat, np.array([2], np.int32))
    p0 = 1.0 / (1.0 + np.exp(-a / math.sqrt(d)))
    assert np.allclose(got[0, :, 1], p0, rtol=0, atol=1e-15), f"{got[0, :, 1]} vs {p0}"
    assert np.allclose(got[0, :, 2], 1.0 - p0, rtol=0, atol=1e-15)
    mask = np.ones(d, bool)
    mask[[1, 2]] = False
    assert np.all(got[0][:, mask] == 0.0)


def check_uniform_keys(o, r: int = 32, d: int = 128) -> None:
    """Identical keys give uniform weights: o is the mean of the reconstructed values."""
    rng = np.random.default_rng(14)
    L = 23
    P_K = si.bases(51, 1, d, r)
    P_V = _identity_basis(d, r)[None]
    k_lat = np.repeat(rng.standard_normal((1, 1, 1, r)), L, axis=2)
    v_lat = rng.standard_normal((1, 1, L, r))
    q = rng.standard_normal((1, 2, d))
    got = o.decode(q, P_K, P_V, k_lat, v_lat, np.array([L], np.int32))
    want = np.zeros((1, 2, d))
    want[0, :, :r] = v_lat[0, 0].mean(axis=0)
    assert _rel_err(got, want) <= 1e-13


def check_token_order_invariance(o, r: int = 48, d: int = 128) -> None:
    """Permuting the cache rows (keys and values together) does not change the output."""
    rng = np.random.default_rng(15)
    L = 31
    P_K = si.bases(61, 2, d, r)
    P_V = si.bases(62, 2, d, r)
    k_lat = rng.standard_normal((1, 2, L, r))
    v_lat = rng.standard_normal((1, 2, L, r))
    q = 3.0 * rng.standard_normal((1, 4, d))
    lens = np.array([L], np.int32)
    perm = rng.permutation(L)
    a = o.decode(q, P_K, P_V, k_lat, v_lat, lens)
    b = o.decode(q, P_K, P_V, k_lat[:, :, perm], v_lat[:, :, perm], lens)
    assert _rel_err(b, a) <= 1e-12


def check_empty_sequence(o, r: int = 64, d: int = 128) -> None:
    """Length 0 attends to nothing: output exactly zero (and finite)."""
    rng = np.random.default_rng(16)
    P = si.bases(71, 1, d, r)
    got = o.decode(rng.standard_normal((2, 4, d)), P, P, rng.standard_normal((2, 1, 8, r)),
                   rng.standard_normal((2, 1, 8, r)), np.array([0, 3], np.int32))
    assert np.all(got[0] == 0.0)
    assert np.all(np.isfinite(got[1])) and np.any(got[1] != 0.0)


# ----------------------------------------------------------------------------- latent decode

def check_latent_is_sdpa_on_latent_rows(o, q_scale: float = 1.0, tol: float = 1e-12) -> None:
    """The latent decode is softmax attention over the latent rows themselves, with the
    score scale 1/sqrt(d) of the full head dimension (torch SDPA, float64, explicit scale)."""
    d = 128
    B, Hq, Hkv, L_max, rK, rV = 2, 8, 2, 40, 48, 32
    lens = np.array([37, 5], dtype=np.int32)
    rng = np.random.default_rng(17)
    q = q_scale * rng.standard_normal((B, Hq, rK))
    k = rng.standard_normal((B, Hkv, L_max, rK))
    v = rng.standard_normal((B, Hkv, L_max, rV))
    got = o.decode_latent(q, k, v, lens, d=d)
    want = np.zeros((B, Hq, rV))
    for b in range(B):
        L = int(lens[b])
        oq = F.scaled_dot_product_attention(
            torch.from_numpy(q[b][None, :, None, :]),
            torch.from_numpy(np.ascontiguousarray(k[b][None, :, :L])),
            torch.from_numpy(np.ascontiguousarray(v[b][None, :, :L])),
            scale=1.0 / math.sqrt(d), enable_gqa=True)
        want[b] = oq[0, :, 0, :].numpy()
    assert np.all(np.isfinite(got)), "non-finite output"
    err = _rel_err(got, want)
    assert err <= tol, f"latent decode differs from attention over the latent rows: {err}"


def check_latent_folding_identity(o, d: int = 128) -> None:
    """Folding the bases into the weights changes nothing: decode_latent(q P_K) P_V^T equals
    decode(q) over the same cache (associativity of the products)."""
    rng = np.random.default_rng(18)
    B, Hq, Hkv, L, rK, rV = 2, 8, 4, 33, 64, 48
    q = rng.standard_normal((B, Hq, d))
    P_K = si.bases(81, Hkv, d, rK)
    P_V = si.bases(82, Hkv, d, rV)
    k = rng.standard_normal((B, Hkv, L, rK))
    v = rng.standard_normal((B, Hkv, L, rV))
    lens = np.array([L, 12], np.int32)
    G = Hq // Hkv
    q_lat = np.stack([np.stack([q[b, h] @ P_K[h // G] for h in range(Hq)]) for b in range(B)])
    o_lat = o.decode_latent(q_lat, k, v, lens, d=d)
    got = np.stack([np.stack([o_lat[b, h] @ P_V[h // G].T for h in range(Hq)]) for b in range(B)])
    want = o.decode(q, P_K, P_V, k, v, lens)
    assert _rel_err(got, want) <= 1e-12


def check_latent_edges(o, r: int = 32) -> None:
    """Length 0 gives exactly 0; length 1 gives exactly the one value row."""
    rng = np.random.default_rng(19)
    k = rng.standard_normal((2, 1, 6, r))
    v = rng.standard_normal((2, 1, 6, 2 * r))
    got = o.decode_latent(7.0 * rng.standard_normal((2, 3, r)), k, v, np.array([0, 1], np.int32))
    assert np.all(got[0] == 0.0)
    assert np.array_equal(got[1], np.repeat(v[1, 0, :1], 3, axis=0))


# ----------------------------------------------------------------------------- paged layout

def check_paged_layout(o) -> None:
    """gather_pages inverts a scatter of a known contiguous cache into shuffled pages, and
    token t of sequence b comes from page block_table[b][t // page_size], row t % page_size."""
    rng = np.random.default_rng(20)
    B, Hkv, ps, r, max_pages = 3, 2, 64, 16, 4
    lens = np.array([256, 70, 0], np.int32)
    cont = rng.standard_normal((B, Hkv, max_pages * ps, r))
    perm = rng.permutation(B * max_pages)
    bt = perm.reshape(B, max_pages).astype(np.int32)
    pages = np.zeros((B * max_pages, Hkv, ps, r))
    for b in range(B):
        for j in range(max_pages):
            pages[bt[b, j]] = cont[b, :, j * ps:(j + 1) * ps]
    import oracle  # gather_pages is plain indexing in the Python module (no C part)
    got = oracle.gather_pages(pages, bt, lens, max_pages * ps)
    for b in range(B):
        assert np.array_equal(got[b, :, :lens[b]], cont[b, :, :lens[b]])
        assert np.all(got[b, :, lens[b]:] == 0)
    # one hand-picked token: sequence 1, token 69 -> page bt[1][1], row 5
    assert np.array_equal(got[1, :, 69], pages[bt[1, 1], :, 5])


# ----------------------------------------------------------------------------- int8 rows

def check_quantize_rows(o) -> None:
    """Closed forms of the per-row int8 form: the largest magnitude maps to +-127 exactly;
    a zero row is scale 0 and codes 0; codes are odd-symmetric; halfway cases round to even;
    every element is within half a step (plus the fp32 division's rounding) of its code."""
    import oracle
    rng = np.random.default_rng(21)
    x = oracle.round_bf16(rng.standard_normal((64, 48)) * rng.uniform(0.01, 10, (64, 1)))
    q, s = oracle.quantize_rows(x)
    assert q.dtype == np.int8 and s.dtype == np.float32
    amax_idx = np.argmax(np.abs(x), axis=1)
    assert np.all(np.abs(q[np.arange(64), amax_idx]) == 127)
    assert np.all(np.sign(q[np.arange(64), amax_idx]) == np.sign(x[np.arange(64), amax_idx]))
    err = np.abs(x - oracle.dequantize_rows(q, s))
    assert np.all(err <= 0.5 * s[:, None] * (1 + 2.0 ** -22) + np.abs(x) * 2.0 ** -23)
    qn, sn = oracle.quantize_rows(-x)
    assert np.array_equal(qn, -q) and np.array_equal(sn, s)
    z, zs = oracle.quantize_rows(np.zeros((2, 16)))
    assert np.all(z == 0) and np.all(zs == 0)
    # row max 127 gives scale exactly 1: x = k + 0.5 rounds to the even neighbour
    row = np.array([[127.0, 2.5, 3.5, -2.5, -0.5, 0.5, 1.5, 126.5]])
    qr, sr = oracle.quantize_rows(row)
    assert sr[0] == 1.0
    assert qr[0].tolist() == [127, 2, 4, -2, 0, 0, 2, 126]


def check_quantize_rows_q4(o) -> None:
    """The 4-bit form: the largest magnitude maps to +-7 exactly; codes stay in [-7, 7]; halfway
    cases round to even; every element is within half a step of its code; and the packing puts
    column 2j in the low and 2j + 1 in the high nibble of byte j (hand-packed bytes below),
    round-tripping every code of [-8, 7]."""
    import oracle
    rng = np.random.default_rng(22)
    x = oracle.round_bf16(rng.standard_normal((64, 64)) * rng.uniform(0.01, 10, (64, 1)))
    q, s = oracle.quantize_rows(x, qmax=7)
    assert q.dtype == np.int8 and s.dtype == np.float32
    assert q.min() >= -7 and q.max() <= 7
    amax_idx = np.argmax(np.abs(x), axis=1)
    assert np.all(np.abs(q[np.arange(64), amax_idx]) == 7)
    err = np.abs(x - oracle.dequantize_rows(q, s))
    assert np.all(err <= 0.5 * s[:, None] * (1 + 2.0 ** -22) + np.abs(x) * 2.0 ** -23)
    # row max 7 gives scale exactly 1: x = k + 0.5 rounds to the even neighbour
    row = np.array([[7.0, 2.5, 3.5, -2.5, -0.5, 0.5, 1.5, -6.5]])
    qr, sr = oracle.quantize_rows(row, qmax=7)
    assert sr[0] == 1.0
    assert qr[0].tolist() == [7, 2, 4, -2, 0, 0, 2, -6]
    # packing: (lo, hi) = (7, 2) -> 0x27; (4, -2) -> 0xE4; (0, 0) -> 0x00; (2, -6) -> 0xA2
    packed = oracle.pack_q4(qr)
    assert packed.dtype == np.uint8 and packed.shape == (1, 4)
    assert packed[0].tolist() == [0x27, 0xE4, 0x00, 0xA2]
    allc = np.arange(-8, 8, dtype=np.int8)
    grid = np.stack(np.meshgrid(allc, allc, indexing="ij"), -1).reshape(-1, 2)  # every (lo, hi)
    assert np.array_equal(oracle.unpack_q4(oracle.pack_q4(grid)), grid)
    assert sorted(oracle.pack_q4(grid)[:, 0].tolist()) == list(range(256))
    assert np.array_equal(oracle.unpack_q4(oracle.pack_q4(q)), q)


# ----------------------------------------------------------------------------- compression

def check_compress_identity_basis(o, r: int = 48, d: int = 128) -> None:
    """P = [I_r; 0]: the stored latent is exactly the first r coordinates of each bf16 row."""
    rng = np.random.default_rng(17)
    x = si.bf16_to_f64(si.to_bf16(rng.standard_normal((19, d))))
    y = o.project(x, _identity_basis(d, r), round_to_bf16=True)
    assert np.array_equal(y, x[:, :r])


def check_compress_matches_exact_product(o, r: int = 64, d: int = 128) -> None:
    """Unrounded compression equals x.P to fp64 round-off; rounded is its RNE bf16 value."""
    rng = np.random.default_rng(18)
    x = si.bf16_to_f64(si.to_bf16(rng.standard_normal((33, d))))
    P = si.bf16_to_f64(si.to_bf16(si.bases(81, 1, d, r)[0]))
    exact = o.project(x, P, round_to_bf16=False)
    lib = x @ P
    assert _rel_err(exact, lib) <= 1e-14
    rounded = o.project(x, P, round_to_bf16=True)
    ref = torch.from_numpy(exact.astype(np.float32)).to(torch.bfloat16).to(torch.float64).numpy()
    # double rounding fp64 -> fp32 -> bf16 can differ from direct RNE only at near-ties
    ulp = np.exp2(np.floor(np.log2(np.abs(ref) + 1e-300)) - 7)
    assert np.all(np.abs(rounded - ref) <= ulp)
    assert np.mean(rounded == ref) > 0.999


def check_compress_append_bookkeeping(o, r: int = 32, d: int = 128) -> None:
    """Rows land exactly at [len, len+T); other slots are untouched; overflow writes nothing."""
    rng = np.random.default_rng(19)
    B, Hkv, T, L_max = 3, 2, 3, 10
    lens = np.array([0, 7, 8], np.int32)   # the second fills the cache exactly, the last overflows
    k_new = si.bf16_to_f64(si.to_bf16(rng.standard_normal((B, Hkv, T, d))))
    v_new = si.bf16_to_f64(si.to_bf16(rng.standard_normal((B, Hkv, T, d))))
    P = _identity_basis(d, r)[None].repeat(Hkv, axis=0)
    canary = 12345.0
    k_lat = np.full((B, Hkv, L_max, r), canary)
    v_lat = np.full((B, Hkv, L_max, r), -canary)
    kl, vl, new_lens, nbad = o.compress_append(k_new, v_new, P, P, k_lat, v_lat, lens)
    assert nbad == 1
    assert new_lens.tolist() == [3, 10, 8]
    for b in range(B):
        for h in range(Hkv):
            if b < 2:
                s = int(lens[b])
                assert np.array_equal(kl[b, h, s:s + T], k_new[b, h, :, :r])
                assert np.array_equal(vl[b, h, s:s + T], v_new[b, h, :, :r])
                keep = np.ones(L_max, bool)
                keep[s:s + T] = False
            else:
                keep = np.ones(L_max, bool)
            assert np.all(kl[b, h, keep] == canary)
            assert np.all(vl[b, h, keep] == -canary)


# ----------------------------------------------------------------------------- joint value latent
#
# STAR-KV technical summary, "Metodologia" item 2: values decomposed jointly over the
# concatenated heads, keys per head; the value reconstruction is absorbed into the output
# projection.  The oracle's joint-value calls are layout over decode / decode_latent / project;
# these pins fix the layout (concatenation order, the block of P_VJ each head reads, the shared
# latent) against plain attention and against the per-head form.

def _block_diag(P):
    """[Hkv][d][r] -> the (Hkv*d) x (Hkv*r) block-diagonal matrix with block g = P[g]."""
    Hkv, d, r = P.shape
    out = np.zeros((Hkv * d, Hkv * r))
    for g in range(Hkv):
        out[g * d:(g + 1) * d, g * r:(g + 1) * r] = P[g]
    return out


def check_joint_v_full_rank_is_plain_attention(o, d: int = 32, tol: float = 1e-12) -> None:
    """rK = d and rV = Hkv*d: both reconstructions are exact, so compress-then-decode with a
    joint value basis is plain attention on the original rows (torch SDPA, float64).  A
    concatenation order that differs between compression and reconstruction fails here."""
    B, Hq, Hkv, L_max, T = 2, 6, 3, 24, 24
    lens = np.array([24, 7], dtype=np.int32)
    rng = np.random.default_rng(23)
    K = rng.standard_normal((B, Hkv, T, d))
    V = rng.standard_normal((B, Hkv, T, d))
    q = rng.standard_normal((B, Hq, d))
    P_K = si.bases(24, Hkv, d, d)
    P_VJ = si.bases(25, 1, Hkv * d, Hkv * d)[0]
    k_lat, v_joint, new_lens, nbad = o.compress_append_joint_v(
        K, V, P_K, P_VJ, np.zeros((B, Hkv, L_max, d)), np.zeros((B, L_max, Hkv * d)),
        np.zeros(B, np.int32), round_to_bf16=False)
    assert nbad == 0 and new_lens.tolist() == [T, T]
    got = o.decode_joint_v(q, P_K, P_VJ, k_lat, v_joint, lens)
    want = _sdpa_reference(q, K, V, lens)
    assert np.all(np.isfinite(got)), "non-finite output"
    err = _rel_err(got, want)
    assert err <= tol, f"joint values at full rank differ from plain attention: {err}"


def check_joint_v_block_diagonal_is_per_head(o, r: int = 16, d: int = 128) -> None:
    """P_VJ = blockdiag(P_V[0], ..., P_V[Hkv-1]): the joint latent of a token is the per-head
    latents side by side, and decode_joint_v equals the per-head decode over them (the
    products with the zero blocks add exact zeros, so the caches agree bit for bit)."""
    B, Hq, Hkv, L_max, T = 2, 8, 4, 12, 9
    rng = np.random.default_rng(26)
    k_new = si.bf16_to_f64(si.to_bf16(rng.standard_normal((B, Hkv, T, d))))
    v_new = si.bf16_to_f64(si.to_bf16(rng.standard_normal((B, Hkv, T, d))))
    P_K = si.bases(27, Hkv, d, 24)
    P_V = si.bases(28, Hkv, d, r)
    lens0 = np.array([0, 3], np.int32)
    kj, vj, lj, _ = o.compress_append_joint_v(k_new, v_new, P_K, _block_diag(P_V),
                                              np.zeros((B, Hkv, L_max, 24)),
                                              np.zeros((B, L_max, Hkv * r)), lens0)
    kp, vp, lp, _ = o.compress_append(k_new, v_new, P_K, P_V, np.zeros((B, Hkv, L_max, 24)),
                                      np.zeros((B, Hkv, L_max, r)), lens0)
    assert np.array_equal(lj, lp) and np.array_equal(kj, kp)
    for g in range(Hkv):
        assert np.array_equal(vj[:, :, g * r:(g + 1) * r], vp[:, g])
    q = rng.standard_normal((B, Hq, d))
    got = o.decode_joint_v(q, P_K, _block_diag(P_V), kj, vj, lj)
    want = o.decode(q, P_K, P_V, kp, vp, lp)
    assert _rel_err(got, want) <= 1e-14


def check_joint_v_latent_folding(o, d: int = 64) -> None:
    """Folding: decode_latent_joint_v(q P_K[g]) followed by block g of P_VJ equals
    decode_joint_v(q) (associativity of the products)."""
    rng = np.random.default_rng(29)
    B, Hq, Hkv, L, rK, rV = 2, 8, 2, 21, 32, 40
    q = rng.standard_normal((B, Hq, d))
    P_K = si.bases(30, Hkv, d, rK)
    P_VJ = si.bases(31, 1, Hkv * d, rV)[0]
    k = rng.standard_normal((B, Hkv, L, rK))
    v = rng.standard_normal((B, L, rV))
    lens = np.array([L, 4], np.int32)
    G = Hq // Hkv
    q_lat = np.stack([np.stack([q[b, h] @ P_K[h // G] for h in range(Hq)]) for b in range(B)])
    o_lat = o.decode_latent_joint_v(q_lat, k, v, lens, d=d)
    blk = lambda g: P_VJ[g * d:(g + 1) * d]
    got = np.stack([np.stack([blk(h // G) @ o_lat[b, h] for h in range(Hq)]) for b in range(B)])
    want = o.decode_joint_v(q, P_K, P_VJ, k, v, lens)
    assert _rel_err(got, want) <= 1e-12


def check_joint_v_edges(o, d: int = 16) -> None:
    """One token: every query head of KV head g returns block g of v_joint[0] . P_VJ^T (its
    softmax weight is 1); the latent form returns v_joint[0] itself.  Length 0 gives 0."""
    rng = np.random.default_rng(32)
    Hkv, Hq, rK, rV = 3, 6, 8, 12
    P_K = si.bases(33, Hkv, d, rK)
    P_VJ = si.bases(34, 1, Hkv * d, rV)[0]
    k = rng.standard_normal((2, Hkv, 5, rK))
    v = rng.standard_normal((2, 5, rV))
    lens = np.array([0, 1], np.int32)
    got = o.decode_joint_v(5.0 * rng.standard_normal((2, Hq, d)), P_K, P_VJ, k, v, lens)
    assert np.all(got[0] == 0.0)
    full = P_VJ @ v[1, 0]                      # the reconstructed concatenation, Hkv*d long
    G = Hq // Hkv
    for h in range(Hq):
        g = h // G
        assert np.allclose(got[1, h], full[g * d:(g + 1) * d], rtol=0, atol=1e-14)
    lat = o.decode_latent_joint_v(rng.standard_normal((2, Hq, rK)), k, v, lens, d=d)
    assert np.all(lat[0] == 0.0)
    assert np.array_equal(lat[1], np.repeat(v[1, :1], Hq, axis=0))


def check_joint_v_compress_bookkeeping(o, d: int = 16) -> None:
    """Joint rows land exactly at [len, len+T) of the sequence's value latent, keys per head
    as in compress_append; a sequence that would overflow is left untouched."""
    rng = np.random.default_rng(35)
    B, Hkv, T, L_max, rK = 3, 2, 3, 10, 8
    lens = np.array([0, 7, 8], np.int32)
    k_new = si.bf16_to_f64(si.to_bf16(rng.standard_normal((B, Hkv, T, d))))
    v_new = si.bf16_to_f64(si.to_bf16(rng.standard_normal((B, Hkv, T, d))))
    P_K = np.repeat(_identity_basis(d, rK)[None], Hkv, axis=0)
    P_VJ = np.eye(Hkv * d)                      # the stored latent is the concatenation itself
    kl, vj, new_lens, nbad = o.compress_append_joint_v(
        k_new, v_new, P_K, P_VJ, np.full((B, Hkv, L_max, rK), 7.0),
        np.full((B, L_max, Hkv * d), -7.0), lens)
    assert nbad == 1 and new_lens.tolist() == [3, 10, 8]
    for b in range(2):
        s = int(lens[b])
        for t in range(T):
            assert np.array_equal(vj[b, s + t], np.concatenate([v_new[b, g, t] for g in range(Hkv)]))
            assert np.array_equal(kl[b, :, s + t], k_new[b, :, t, :rK])
        keep = np.ones(L_max, bool)
        keep[s:s + T] = False
        assert np.all(vj[b, keep] == -7.0) and np.all(kl[b, :, keep] == 7.0)
    assert np.all(vj[2] == -7.0) and np.all(kl[2] == 7.0)


ALL_ORACLE_CHECKS = {
    "round_bf16_matches_torch": check_round_bf16_matches_torch,
    "round_bf16_edges": check_round_bf16_edges,
    "full_rank_is_plain_attention": check_full_rank_is_plain_attention,
    # scores in the hundreds: exp() overflows unless the maximum is subtracted first
    "full_rank_large_scores": lambda o: check_full_rank_is_plain_attention(o, q_scale=400.0,
                                                                           tol=1e-10),
    "tiny_compressed_is_sdpa_on_reconstructed_rows":
        check_tiny_compressed_is_sdpa_on_reconstructed_rows,
    "gauge_invariance": check_gauge_invariance,
    "single_token": check_single_token,
    "two_tokens": check_two_tokens,
    "uniform_keys": check_uniform_keys,
    "token_order_invariance": check_token_order_invariance,
    "empty_sequence": check_empty_sequence,
    "latent_is_sdpa_on_latent_rows": check_latent_is_sdpa_on_latent_rows,
    # scores past 709, where exp() overflows: the latent path must subtract the maximum too
    "latent_large_scores": lambda o: check_latent_is_sdpa_on_latent_rows(o, q_scale=2000.0,
                                                                         tol=1e-10),
    "latent_folding_identity": check_latent_folding_identity,
    "latent_edges": check_latent_edges,
    "paged_layout": check_paged_layout,
    "quantize_rows": check_quantize_rows,
    "quantize_rows_q4": check_quantize_rows_q4,
    "compress_identity_basis": check_compress_identity_basis,
    "compress_matches_exact_product": check_compress_matches_exact_product,
    "compress_append_bookkeeping": check_compress_append_bookkeeping,
    "joint_v_full_rank_is_plain_attention": check_joint_v_full_rank_is_plain_attention,
    "joint_v_block_diagonal_is_per_head": check_joint_v_block_diagonal_is_per_head,
    "joint_v_latent_folding": check_joint_v_latent_folding,
    "joint_v_edges": check_joint_v_edges,
    "joint_v_compress_bookkeeping": check_joint_v_compress_bookkeeping,
}
