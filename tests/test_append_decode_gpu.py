"""The fused step stief_append_decode (CUDA, through the C ABI) against the oracle's append
followed by its decode (StiefAttention technical summary, "Mecanismo Central" item 5).

Output: within the decode tolerance of the oracle run on the grown cache.  The appended
latent rows: the bf16 rounding of a tensor-core fp32 sum, so within half a bf16 ulp plus
the fp32 dot-product error bound of the exact product (taken with a unit roundoff of
2^-23, as the tensor core's adder may truncate), and nearly all equal to the oracle's
rounding of the exact product.  Lengths and untouched cache rows: bit-exact.
"""
import numpy as np
import pytest
import torch

import decode_attention_stief_b200 as stief
import oracle
import stief_inputs as si
from gpu_util import DECODE_TOL, bf16_ulp, decode_error, f64, make_decode_case

pytestmark = pytest.mark.gpu

GAMMA_128_TC = 128 * 2.0 ** -23 / (1 - 128 * 2.0 ** -23)


def _latent_ok(got_bits, x, P):
    """Rows of got = RNE_bf16(fp32 sum of x . P): bound check; returns the exact-match count."""
    g = f64(got_bits)
    exact = oracle.project(x, P, round_to_bf16=False)
    want = oracle.project(x, P, round_to_bf16=True)
    bound = 0.5 * bf16_ulp(np.maximum(np.abs(g), np.abs(exact))) + \
        GAMMA_128_TC * (np.abs(x) @ np.abs(P))
    err = np.abs(g - exact)
    assert np.all(err <= bound), f"max excess {np.max(err - bound)}"
    return int(np.sum(g == want)), g.size


def _case(B, Hq, Hkv, rK, rV, L_max, lens, seed, poison_tail=True):
    d = 128
    q = si.queries(seed, B, Hq, d)
    P_K, P_V = si.bases_bf16(seed, Hkv, d, rK, rV)
    k_lat = si.latent_cache(seed, B, Hkv, L_max, rK, 0)
    v_lat = si.latent_cache(seed, B, Hkv, L_max, rV, 1)
    if poison_tail:  # rows at and past the length hold NaN: only the append may write them
        for b, L in enumerate(lens):
            k_lat[b, :, L:] = float("nan")
            v_lat[b, :, L:] = float("nan")
    kn, vn = si.full_kv(seed + 1, B, Hkv, 1, d)
    return q, kn[:, :, 0], vn[:, :, 0], P_K, P_V, k_lat, v_lat


def _run(q, kn, vn, P_K, P_V, k_lat, v_lat, lens, max_seq_len, num_splits=0, expect_status=0,
         ws=None):
    dev = torch.device("cuda")
    q, kn, vn, P_K, P_V, k_lat, v_lat = (x.to(dev).contiguous() for x in (q, kn, vn, P_K, P_V, k_lat, v_lat))
    lens_t = torch.as_tensor(np.asarray(lens, np.int32)).to(dev)
    B, Hq, d = q.shape
    out = torch.full((B, Hq, d), float("nan"), dtype=torch.bfloat16, device=dev)
    if ws is None:
        ws = stief.workspace_for(B, Hq, P_K.shape[0], P_V.shape[2], max_seq_len)
    status = torch.zeros(1, dtype=torch.int32, device=dev)
    stief.stief_append_decode(q, kn, vn, P_K, P_V, k_lat, v_lat, lens_t, out, ws, max_seq_len,
                              num_splits=num_splits, dev_status=status)
    st = stief.stief_read_device_status(status)
    assert st == expect_status, f"device status {st:#x}"
    return out.cpu(), k_lat.cpu(), v_lat.cpu(), lens_t.cpu().numpy(), ws


def _oracle_step(q, kn, vn, P_K, P_V, k_lat, v_lat, lens):
    """oracle append (T = 1) then oracle decode; returns (out, k_lat, v_lat, lens)."""
    k2, v2, l2, nover = oracle.compress_append(f64(kn)[:, :, None], f64(vn)[:, :, None], f64(P_K),
                                               f64(P_V), f64(k_lat), f64(v_lat),
                                               np.asarray(lens, np.int32))
    return oracle.decode(f64(q), f64(P_K), f64(P_V), k2, v2, l2), k2, v2, l2, nover


def _check(case, lens, max_seq_len, num_splits=0):
    q, kn, vn, P_K, P_V, k_lat, v_lat = case
    got, gk, gv, glens, _ = _run(q, kn, vn, P_K, P_V, k_lat, v_lat, lens, max_seq_len, num_splits)
    want, wk, wv, wlens, _ = _oracle_step(q, kn, vn, P_K, P_V, k_lat, v_lat, lens)
    assert glens.tolist() == wlens.tolist() == [L + 1 for L in lens]
    err = decode_error(got, want)
    assert err <= DECODE_TOL, f"max|err| / ||o||_inf = {err:.3e}"
    same = total = 0
    for b, L in enumerate(lens):
        for h in range(P_K.shape[0]):
            s1, n1 = _latent_ok(gk[b, h, L:L + 1], f64(kn[b, h])[None], f64(P_K[h]))
            s2, n2 = _latent_ok(gv[b, h, L:L + 1], f64(vn[b, h])[None], f64(P_V[h]))
            same, total = same + s1 + s2, total + n1 + n2
    assert same >= 0.98 * total, f"{same}/{total} latent elements equal the oracle's rounding"
    # every other row is bit-for-bit what it was (the poisoned tail included)
    for b, L in enumerate(lens):
        for x_got, x0 in ((gk, k_lat), (gv, v_lat)):
            gb = x_got[b].view(torch.int16).clone()
            ob = x0[b].view(torch.int16).clone()
            gb[:, L] = 0
            ob[:, L] = 0
            assert torch.equal(gb, ob)
    return err


@pytest.mark.parametrize("rK,rV", [(64, 64), (32, 48), (16, 16), (96, 64), (48, 128)])
def test_append_decode_matches_oracle(rK, rV):
    lens = [0, 31, 64, 700]
    case = _case(4, 32, 8, rK, rV, 760, lens, 3000 + rK + rV)
    _check(case, lens, max_seq_len=720)


@pytest.mark.parametrize("G", [1, 2, 3, 4, 8])
def test_append_decode_gqa_groups(G):
    lens = [129, 1]
    case = _case(2, 2 * G, 2, 64, 64, 300, lens, 3100 + G)
    _check(case, lens, max_seq_len=260)


@pytest.mark.parametrize("S", [1, 2, 5, 8])
def test_append_decode_split_boundaries(S):
    """The new token at the first and last row of a split, of a 32- and a 64-token tile."""
    for lens in ([127, 128], [255, 256], [64 * 5 - 1, 64 * 5]):
        case = _case(2, 8, 2, 32, 32, 1100, lens, 3200 + S + lens[0])
        _check(case, lens, max_seq_len=1024, num_splits=S)


def test_append_decode_full_size_sample():
    """The 32k decode shape (1 sequence, 32/8 heads, ranks 64/64) in the launch configuration
    the benchmark uses; the oracle checks a sample of heads, exactly."""
    dev = torch.device("cuda")
    B, Hq, Hkv, d, rK, rV, L0 = 1, 32, 8, 128, 64, 64, 32767
    L_max = L0 + 8
    P_K, P_V = si.bases_bf16(3300, Hkv, d, rK, rV)
    k_lat = si.latent_cache_torch(3301, B, Hkv, L_max, rK, 0, dev)
    v_lat = si.latent_cache_torch(3302, B, Hkv, L_max, rV, 1, dev)
    q = si.queries_torch(3303, B, Hq, d, dev)
    kn = torch.randn((B, Hkv, d), device=dev).to(torch.bfloat16)
    vn = torch.randn((B, Hkv, d), device=dev).to(torch.bfloat16)
    lens = [L0]
    got, gk, gv, glens, _ = _run(q, kn, vn, P_K, P_V, k_lat, v_lat, lens, L_max)
    assert glens.tolist() == [L0 + 1]
    for h in (0, 5):
        qh = q[:, 4 * h:4 * h + 4].cpu()
        want = oracle.decode(f64(qh), f64(P_K[h:h + 1]), f64(P_V[h:h + 1]),
                             f64(gk[:, h:h + 1]), f64(gv[:, h:h + 1]), np.array([L0 + 1], np.int32))
        err = decode_error(got[:, 4 * h:4 * h + 4], want)
        assert err <= DECODE_TOL
        _latent_ok(gk[0, h, L0:L0 + 1], f64(kn[0, h].cpu())[None], f64(P_K[h]))


def test_append_decode_capacity_overflow():
    """A full cache is not appended to: the status bit is set, the length and every row stay,
    and the output attends over the rows present."""
    lens = [40, 48]
    case = _case(2, 8, 2, 64, 64, 48, lens, 3400, poison_tail=False)
    q, kn, vn, P_K, P_V, k_lat, v_lat = case
    got, gk, gv, glens, _ = _run(q, kn, vn, P_K, P_V, k_lat, v_lat, lens, 48,
                                 expect_status=stief.DEV_CAPACITY_OVERFLOW)
    assert glens.tolist() == [41, 48]
    assert torch.equal(gk[1].view(torch.int16), k_lat[1].view(torch.int16))
    assert torch.equal(gv[1].view(torch.int16), v_lat[1].view(torch.int16))
    want1 = oracle.decode(f64(q[1:]), f64(P_K), f64(P_V), f64(k_lat[1:]), f64(v_lat[1:]),
                          np.array([48], np.int32))
    assert decode_error(got[1:], want1) <= DECODE_TOL


def test_append_decode_consecutive_steps_and_counters():
    """Three steps in a row on one workspace equal three oracle steps, and the workspace
    counters are back at zero after each."""
    lens = [300, 17, 0]
    q, kn0, vn0, P_K, P_V, k_lat, v_lat = _case(3, 8, 2, 48, 32, 400, lens, 3500)
    dev = torch.device("cuda")
    gk, gv, glens = k_lat, v_lat, list(lens)
    wk, wv, wlens = f64(k_lat), f64(v_lat), np.asarray(lens, np.int32)
    ws = None
    for step in range(3):
        kn, vn = si.full_kv(3600 + step, 3, 2, 1, 128)
        kn, vn = kn[:, :, 0], vn[:, :, 0]
        got, gk, gv, glens_np, ws = _run(q, kn, vn, P_K, P_V, gk, gv, glens, 400, ws=ws)
        glens = glens_np.tolist()
        wk, wv, wlens, _ = oracle.compress_append(f64(kn)[:, :, None], f64(vn)[:, :, None],
                                                  f64(P_K), f64(P_V), wk, wv, wlens)
        want = oracle.decode(f64(q), f64(P_K), f64(P_V), wk, wv, wlens)
        assert glens == wlens.tolist()
        assert decode_error(got, want) <= DECODE_TOL
        counters = ws[: (3 * 2 * 1 + 3) * 4].view(torch.int32).cpu()
        assert torch.all(counters == 0), counters


def test_append_decode_equals_two_calls():
    """The fused step and the two separate calls give the same lengths, nearly the same rows
    (both round once; the sums may differ in order) and outputs within the decode tolerance."""
    lens = [500, 33]
    q, kn, vn, P_K, P_V, k_lat, v_lat = _case(2, 32, 8, 64, 64, 640, lens, 3700, poison_tail=False)
    got, gk, gv, glens, _ = _run(q, kn, vn, P_K, P_V, k_lat, v_lat, lens, 640)
    dev = torch.device("cuda")
    k2, v2 = k_lat.to(dev).contiguous(), v_lat.to(dev).contiguous()
    l2 = torch.as_tensor(np.asarray(lens, np.int32)).to(dev)
    stief.stief_compress_append(kn[:, :, None].to(dev).contiguous(), vn[:, :, None].to(dev).contiguous(),
                                P_K.to(dev), P_V.to(dev), k2, v2, l2)
    out2 = torch.empty_like(q).to(dev)
    ws = stief.workspace_for(2, 32, 8, 64, 640)
    stief.stief_decode_attention(q.to(dev), P_K.to(dev), P_V.to(dev), k2, v2, l2, out2, ws, 640)
    assert glens.tolist() == l2.cpu().tolist()
    ulps = (f64(gk) - f64(k2.cpu())) / bf16_ulp(f64(k2.cpu()))
    assert np.max(np.abs(ulps)) <= 1.0
    ref = f64(out2.cpu())
    assert np.max(np.abs(f64(got) - ref)) <= DECODE_TOL * np.max(np.abs(ref))


@pytest.mark.parametrize("num_splits", [0, 6])
def test_back_to_back_steps_without_host_sync(num_splits):
    """Fused steps queued back to back on the same caches (nothing between them, no host
    synchronisation) equal the oracle's steps in sequence.  Each launch requests its first
    tiles before its dependency wait, while the launch before it may still be appending the
    row just below the new length; the kernel reads that row again after the wait.  A latent
    decode queued right after the last step sees the grown caches as well."""
    dev = torch.device("cuda")
    lens = [700, 129, 0]
    B, Hq, Hkv, rK, rV, L_max = 3, 8, 2, 64, 64, 800
    q, _, _, P_K, P_V, k_lat, v_lat = _case(B, Hq, Hkv, rK, rV, L_max, lens, 3800)
    qd, Pk, Pv, gk, gv = (x.to(dev).contiguous() for x in (q, P_K, P_V, k_lat, v_lat))
    lens_t = torch.as_tensor(np.asarray(lens, np.int32)).to(dev)
    ws = stief.workspace_for(B, Hq, Hkv, rV, L_max)
    status = torch.zeros(1, dtype=torch.int32, device=dev)
    steps = []
    for step in range(5):
        kn, vn = si.full_kv(3900 + step, B, Hkv, 1, 128)
        kn, vn = kn[:, :, 0].contiguous(), vn[:, :, 0].contiguous()
        out = torch.full((B, Hq, 128), float("nan"), dtype=torch.bfloat16, device=dev)
        stief.stief_append_decode(qd, kn.to(dev), vn.to(dev), Pk, Pv, gk, gv, lens_t, out, ws,
                                  L_max, num_splits=num_splits, dev_status=status)
        steps.append((kn, vn, out))
    q_lat = si.queries(3950, B, Hq, rK).to(dev)
    o_lat = torch.empty((B, Hq, rV), dtype=torch.bfloat16, device=dev)
    stief.stief_decode_latent(q_lat, gk, gv, lens_t, o_lat, ws, L_max, num_splits=num_splits,
                              dev_status=status)
    assert stief.stief_read_device_status(status) == 0
    wk, wv, wl = f64(k_lat), f64(v_lat), np.asarray(lens, np.int32)
    for kn, vn, out in steps:
        wk, wv, wl, _ = oracle.compress_append(f64(kn)[:, :, None], f64(vn)[:, :, None],
                                               f64(P_K), f64(P_V), wk, wv, wl)
        want = oracle.decode(f64(q), f64(P_K), f64(P_V), wk, wv, wl)
        assert decode_error(out.cpu(), want) <= DECODE_TOL
    assert lens_t.cpu().tolist() == wl.tolist() == [L + 5 for L in lens]
    want_l = oracle.decode_latent(f64(q_lat), wk, wv, wl, d=128)
    assert decode_error(o_lat.cpu(), want_l) <= DECODE_TOL


def test_prepared_call_matches_direct_calls():
    """stief.prepare(stief_append_decode, ...) validates once; calling the prepared object
    repeats the same launch.  Three prepared steps and three direct steps on twin caches give
    identical outputs, caches and lengths."""
    B, Hq, Hkv, d, rK, rV, L_max = 2, 16, 4, 128, 64, 64, 512
    dev = torch.device("cuda")
    q, P_K, P_V, k_lat, v_lat = make_decode_case(B, Hq, Hkv, rK, rV, L_max, 9100)
    q, P_K, P_V = q.to(dev), P_K.to(dev), P_V.to(dev)
    caches = [(k_lat.to(dev).clone(), v_lat.to(dev).clone(),
               torch.tensor([300, 41], dtype=torch.int32, device=dev)) for _ in range(2)]
    kn = torch.empty((B, Hkv, d), dtype=torch.bfloat16, device=dev)
    vn = torch.empty_like(kn)
    outs = [torch.empty((B, Hq, d), dtype=torch.bfloat16, device=dev) for _ in range(2)]
    ws = [stief.workspace_for(B, Hq, Hkv, rV, L_max) for _ in range(2)]
    status = torch.zeros(1, dtype=torch.int32, device=dev)
    kl, vl, lens = caches[0]
    prepared = stief.prepare(stief.stief_append_decode, q, kn, vn, P_K, P_V, kl, vl, lens, outs[0],
                             ws[0], max_seq_len=L_max, dev_status=status)
    assert isinstance(prepared, stief.Prepared) and prepared.name == "stief_append_decode"
    g = torch.Generator(device=dev)
    g.manual_seed(9101)
    for step in range(3):
        kn.copy_(torch.randn((B, Hkv, d), generator=g, device=dev).to(torch.bfloat16))
        vn.copy_(torch.randn((B, Hkv, d), generator=g, device=dev).to(torch.bfloat16))
        prepared()
        kl2, vl2, lens2 = caches[1]
        stief.stief_append_decode(q, kn, vn, P_K, P_V, kl2, vl2, lens2, outs[1], ws[1],
                                  max_seq_len=L_max, dev_status=status)
        assert torch.equal(outs[0], outs[1])
    assert stief.stief_read_device_status(status) == 0
    assert torch.equal(caches[0][2], caches[1][2]) and caches[0][2].tolist() == [303, 44]
    assert torch.equal(caches[0][0], caches[1][0]) and torch.equal(caches[0][1], caches[1][1])
