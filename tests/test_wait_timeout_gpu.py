"""Failure detection on the GPU: a bounded wait that runs out reports STIEF_DEV_WAIT_TIMEOUT,
the kernel returns, the context stays usable, and the next call is correct again.

These tests load libstief_testhooks.so, the library built from the same sources with
STIEF_TEST_HOOKS: its bounded waits give up after 50 ms instead of 2 s, and
stief_test_set_stall(bytes) makes every decode planned afterwards expect `bytes` more on its
setup barrier (q, P_K) than any copy delivers, and every tensor-core compress launched
afterwards `bytes` more on each CTA's (or CTA half's) first copy.  That phase then never completes, like a flag
that nothing sets: every wait for it runs out, the kernel reports the timeout, waits (bounded)
for the copies it has in flight and returns.  Nothing faults, traps or waits without a limit.

Recovery follows the header: after a call that reports a timeout the workspace is zeroed
again.  The no-allocation call zeroes the part of its library-owned array it uses before
every launch, which the last test checks by planting stale words there first.
"""
import ctypes

import numpy as np
import pytest
import torch

import decode_attention_stief_b200 as stief
import oracle
from decode_attention_stief_b200 import build as stief_build
from gpu_util import DECODE_TOL, decode_error, f64, make_decode_case, oracle_decode

pytestmark = pytest.mark.gpu

DEV_WAIT_TIMEOUT = 0x2
STALL_BYTES = 16

_vp, _i, _sz = ctypes.c_void_p, ctypes.c_int, ctypes.c_size_t


@pytest.fixture(scope="module")
def hooks():
    path = stief_build.library_file("testhooks")
    lib = ctypes.CDLL(path)
    lib.stief_decode_attention.restype = _i
    lib.stief_decode_attention.argtypes = [_vp] * 8 + [_sz] + [_i] * 9 + [_vp, _vp]
    lib.stief_decode_latent.restype = _i
    lib.stief_decode_latent.argtypes = [_vp] * 6 + [_sz] + [_i] * 9 + [_vp, _vp]
    lib.stief_decode_attention_noalloc.restype = _i
    lib.stief_decode_attention_noalloc.argtypes = [_vp] * 7 + [_i] * 9 + [_vp, _vp]
    for name in ("stief_compress_append", "stief_compress_append_joint_v"):
        fn = getattr(lib, name)
        fn.restype = _i
        fn.argtypes = [_vp] * 7 + [_i] * 7 + [_vp, _vp]
    lib.stief_test_set_stall.restype = None
    lib.stief_test_set_stall.argtypes = [ctypes.c_uint32]
    lib.stief_test_noalloc_scratch.restype = _i
    lib.stief_test_noalloc_scratch.argtypes = [ctypes.POINTER(_vp), ctypes.POINTER(_sz)]
    yield lib
    lib.stief_test_set_stall(0)


def _stream():
    return _vp(torch.cuda.current_stream().cuda_stream)


def _status_word():
    return torch.zeros(1, dtype=torch.int32, device="cuda")


def _read(status) -> int:
    torch.cuda.synchronize()  # the context is still usable after a timed-out launch
    return int(status.item()) & 0xffffffff


def _decode(lib, case, lens, max_seq_len, num_splits, ws, status):
    q, P_K, P_V, k_lat, v_lat = (x.cuda().contiguous() for x in case)
    B, Hq, d = q.shape
    Hkv, _, rK = P_K.shape
    rV = P_V.shape[2]
    lens_t = torch.tensor(lens, dtype=torch.int32, device="cuda")
    out = torch.full((B, Hq, d), float("nan"), dtype=torch.bfloat16, device="cuda")
    code = lib.stief_decode_attention(q.data_ptr(), P_K.data_ptr(), P_V.data_ptr(),
                                      k_lat.data_ptr(), v_lat.data_ptr(), lens_t.data_ptr(),
                                      out.data_ptr(), ws.data_ptr(), ws.numel(), B, Hq, Hkv, d,
                                      rK, rV, k_lat.shape[2], max_seq_len, num_splits,
                                      status.data_ptr(), _stream())
    assert code == 0, stief.stief_status_string(code)
    return out


# (B, Hq, Hkv, rK, rV, L, num_splits): the tagged split merge (96 CTAs at once), the ticket
# merge (a split grid of two waves) and a single split
CASES = [(2, 8, 2, 64, 48, 3000, 0), (16, 32, 8, 64, 64, 1024, 2), (4, 32, 8, 32, 32, 500, 1)]


@pytest.mark.parametrize("B,Hq,Hkv,rK,rV,L,num_splits", CASES)
def test_decode_timeout_reported_then_recovered(hooks, B, Hq, Hkv, rK, rV, L, num_splits):
    case = make_decode_case(B, Hq, Hkv, rK, rV, L, 9100 + B)
    lens = [L - 7 * b for b in range(B)]
    ws = stief.workspace_for(B, Hq, Hkv, rV, L)
    status = _status_word()
    hooks.stief_test_set_stall(STALL_BYTES)
    try:
        _decode(hooks, case, lens, L, num_splits, ws, status)
        assert _read(status) & DEV_WAIT_TIMEOUT, "the stalled launch did not report a timeout"
    finally:
        hooks.stief_test_set_stall(0)
    ws.zero_()  # recovery as documented: zero the workspace after a reported timeout
    status.zero_()
    out = _decode(hooks, case, lens, L, num_splits, ws, status)
    assert _read(status) == 0
    err = decode_error(out.cpu(), oracle_decode(*case, lens))
    assert err <= DECODE_TOL, f"after recovery: max|err| / ||o||_inf = {err:.3e}"


def test_latent_decode_timeout_reported_then_recovered(hooks):
    B, Hq, Hkv, rK, rV, L = 2, 16, 4, 48, 64, 2500
    g = torch.Generator().manual_seed(9200)
    q_lat = torch.randn((B, Hq, rK), generator=g).to(torch.bfloat16).cuda()
    k_lat = torch.randn((B, Hkv, L, rK), generator=g).to(torch.bfloat16).cuda()
    v_lat = torch.randn((B, Hkv, L, rV), generator=g).to(torch.bfloat16).cuda()
    lens = [L, L - 100]
    lens_t = torch.tensor(lens, dtype=torch.int32, device="cuda")
    ws = stief.workspace_for(B, Hq, Hkv, rV, L)
    out = torch.empty((B, Hq, rV), dtype=torch.bfloat16, device="cuda")

    def call(status):
        code = hooks.stief_decode_latent(q_lat.data_ptr(), k_lat.data_ptr(), v_lat.data_ptr(),
                                         lens_t.data_ptr(), out.data_ptr(), ws.data_ptr(),
                                         ws.numel(), B, Hq, Hkv, 128, rK, rV, L, L, 0,
                                         status.data_ptr(), _stream())
        assert code == 0

    status = _status_word()
    hooks.stief_test_set_stall(STALL_BYTES)
    try:
        call(status)
        assert _read(status) & DEV_WAIT_TIMEOUT
    finally:
        hooks.stief_test_set_stall(0)
    ws.zero_()
    status.zero_()
    call(status)
    assert _read(status) == 0
    want = oracle.decode_latent(f64(q_lat), f64(k_lat), f64(v_lat), np.asarray(lens, np.int32),
                                d=128)
    assert decode_error(out.cpu(), want) <= DECODE_TOL


class _DeviceWords:
    """A torch view of device memory at a raw address (no copy, no allocation)."""

    def __init__(self, ptr: int, n: int):
        self.__cuda_array_interface__ = {"shape": (n,), "typestr": "<i8", "data": (ptr, False),
                                         "version": 3}


def test_noalloc_scratch_cleared_before_each_launch(hooks):
    # plant words in the library's own array that a stale call would leave: every 8-byte word
    # a "written" tagged word (tag 1) holding NaN, every ticket counter non-zero
    ptr, nbytes = _vp(), _sz()
    assert hooks.stief_test_noalloc_scratch(ctypes.byref(ptr), ctypes.byref(nbytes)) == 0
    words = torch.as_tensor(_DeviceWords(ptr.value, nbytes.value // 8), device="cuda")
    words.fill_((1 << 32) | 0x7FC00000)
    case = make_decode_case(2, 32, 8, 64, 48, 3000, 9300)
    q, P_K, P_V, k_lat, v_lat = (x.cuda().contiguous() for x in case)
    lens = [3000, 1777]
    lens_t = torch.tensor(lens, dtype=torch.int32, device="cuda")
    out = torch.full((2, 32, 128), float("nan"), dtype=torch.bfloat16, device="cuda")

    def call(status):
        code = hooks.stief_decode_attention_noalloc(
            q.data_ptr(), P_K.data_ptr(), P_V.data_ptr(), k_lat.data_ptr(), v_lat.data_ptr(),
            lens_t.data_ptr(), out.data_ptr(), 2, 32, 8, 128, 64, 48, 3000, 3000, 0,
            status.data_ptr(), _stream())
        assert code == 0

    want = oracle_decode(*case, lens)
    status = _status_word()
    call(status)
    assert _read(status) == 0
    assert decode_error(out.cpu(), want) <= DECODE_TOL
    # a timed-out call, then the next one: nothing to clear by hand
    hooks.stief_test_set_stall(STALL_BYTES)
    try:
        call(status)
        assert _read(status) & DEV_WAIT_TIMEOUT
    finally:
        hooks.stief_test_set_stall(0)
    status.zero_()
    out.fill_(float("nan"))
    call(status)
    assert _read(status) == 0
    assert decode_error(out.cpu(), want) <= DECODE_TOL


# ---------------------------------------------------------------- tensor-core compress kernels

# (joint, B, Hkv, T, rK, rV): the per-head projection (key and value halves of each CTA), the
# joint one with value tiles over CTA pairs (an even Hkv; the pair runs every tile and both of
# its CTAs meet at every cluster barrier after the timeout) and with one CTA per value tile
# (Hkv = 1)
COMPRESS_CASES = [(False, 2, 4, 300, 64, 48), (True, 2, 8, 300, 64, 64), (True, 1, 1, 700, 64, 128),
                  (True, 1, 2, 2600, 32, 64)]


@pytest.mark.parametrize("joint,B,Hkv,T,rK,rV", COMPRESS_CASES)
def test_compress_timeout_reported_then_recovered(hooks, joint, B, Hkv, T, rK, rV):
    """A stalled first copy in every CTA: the tensor-core compress reports the timeout and
    returns (the rows and lengths of that call are undefined); with the lengths put back, the
    next call writes the oracle's rows again."""
    import stief_inputs as si
    d, L_max = 128, T + 40
    k_new, v_new = si.full_kv(9400 + T, B, Hkv, T, d)
    P_K = si.to_bf16(si.bases(9400, Hkv, d, rK))
    if joint:
        P_V = si.to_bf16(si.bases(9401, 1, Hkv * d, rV)[0])
        v_shape = (B, L_max, rV)
        fn = hooks.stief_compress_append_joint_v
    else:
        P_V = si.to_bf16(si.bases(9401, Hkv, d, rV))
        v_shape = (B, Hkv, L_max, rV)
        fn = hooks.stief_compress_append
    kn, vn, pk, pv = (x.cuda().contiguous() for x in (k_new, v_new, P_K, P_V))
    k_lat = torch.zeros((B, Hkv, L_max, rK), dtype=torch.bfloat16, device="cuda")
    v_lat = torch.zeros(v_shape, dtype=torch.bfloat16, device="cuda")
    lens0 = [5 + 11 * b for b in range(B)]
    lens = torch.tensor(lens0, dtype=torch.int32, device="cuda")

    def call(status):
        code = fn(kn.data_ptr(), vn.data_ptr(), pk.data_ptr(), pv.data_ptr(), k_lat.data_ptr(),
                  v_lat.data_ptr(), lens.data_ptr(), B, Hkv, T, d, rK, rV, L_max,
                  status.data_ptr(), _stream())
        assert code == 0, stief.stief_status_string(code)

    status = _status_word()
    hooks.stief_test_set_stall(STALL_BYTES)
    try:
        call(status)
        assert _read(status) & DEV_WAIT_TIMEOUT, "the stalled compress did not report a timeout"
    finally:
        hooks.stief_test_set_stall(0)
    lens.copy_(torch.tensor(lens0, dtype=torch.int32))
    status.zero_()
    call(status)
    assert _read(status) == 0
    assert lens.cpu().tolist() == [L + T for L in lens0]
    # every stored row within half a bf16 ulp of the exact product plus the fp32 accumulation
    # bound K * 2^-23 * sum |x||p| (K = d per head, Hkv * d for the joint values); nothing else
    # written
    gk, gv = f64(k_lat.cpu()), f64(v_lat.cpu())

    def within(got, x, P):
        exact = x @ P
        bound = 2.0 ** -8 * np.abs(exact) + P.shape[0] * 2.0 ** -23 * (np.abs(x) @ np.abs(P))
        return np.all(np.abs(got - exact) <= bound + 1e-30)

    for bb, L in enumerate(lens0):
        for h in range(Hkv):
            assert within(gk[bb, h, L:L + T], f64(k_new[bb, h]), f64(P_K[h]))
            if not joint:
                assert within(gv[bb, h, L:L + T], f64(v_new[bb, h]), f64(P_V[h]))
        if joint:
            x = np.ascontiguousarray(np.transpose(f64(v_new[bb]), (1, 0, 2)).reshape(T, Hkv * d))
            assert within(gv[bb, L:L + T], x, f64(P_V))
        keep = np.ones(L_max, bool)
        keep[L:L + T] = False
        assert not np.any(gk[bb][:, keep])
        assert not np.any(gv[bb][keep] if joint else gv[bb][:, keep])
