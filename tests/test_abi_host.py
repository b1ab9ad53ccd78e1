"""The C-ABI library on the host: it loads, exports every declared symbol, and its
argument checks and planning functions behave (no CUDA call is made here)."""
import ctypes
import os
import re

import pytest

import decode_attention_stief_b200 as stief
from decode_attention_stief_b200 import build as stief_build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "stief.h")

OK, INVALID, ALIGN, CAPACITY, WORKSPACE = 0, 1, 2, 3, 4


@pytest.fixture(scope="module")
def lib():
    stief_build.build_library()
    return stief.library()


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(stief_[a-z_0-9]+)\s*\(", text)))


def test_header_declares_the_entry_points():
    names = declared_functions()
    for required in ("stief_compress_append", "stief_decode_attention",
                     "stief_decode_workspace_bytes", "stief_read_device_status",
                     "stief_status_string"):
        assert required in names


def test_every_declared_symbol_is_exported(lib):
    missing = [n for n in declared_functions() if not hasattr(lib, n)]
    assert not missing, f"not exported: {missing}"


def test_every_declared_call_has_a_binding_of_the_same_name():
    missing = [n for n in declared_functions() if not callable(getattr(stief, n, None))]
    assert not missing, f"no Python binding: {missing}"


def test_only_declared_symbols_are_exported():
    out = os.popen(f"nm -D --defined-only {stief.library_path()}").read()
    exported = set(re.findall(r"\b(stief_[a-z_0-9]+)\b", out))
    assert exported <= set(declared_functions()), exported - set(declared_functions())


def test_status_strings(lib):
    for code, name in stief.STATUS.items():
        assert stief.stief_status_string(code) == name
    assert stief.stief_status_string(99) == "STIEF_ERR_UNKNOWN"


FAKE = 0x10000  # an aligned non-null address; never dereferenced by argument checking


def _decode(lib, **kw):
    a = dict(q=FAKE, P_K=FAKE, P_V=FAKE, k_lat=FAKE, v_lat=FAKE, seq_lens=FAKE, out=FAKE,
             ws=FAKE, ws_bytes=1 << 40, B=1, Hq=32, Hkv=8, d=128, rK=64, rV=64, L_max=1024,
             max_seq_len=1024, num_splits=0)
    a.update(kw)
    return lib.stief_decode_attention(a["q"], a["P_K"], a["P_V"], a["k_lat"], a["v_lat"],
                                      a["seq_lens"], a["out"], a["ws"], a["ws_bytes"], a["B"],
                                      a["Hq"], a["Hkv"], a["d"], a["rK"], a["rV"], a["L_max"],
                                      a["max_seq_len"], a["num_splits"], None, None)


def _compress(lib, **kw):
    a = dict(k=FAKE, v=FAKE, P_K=FAKE, P_V=FAKE, kl=FAKE, vl=FAKE, sl=FAKE, B=1, Hkv=8, T=1,
             d=128, rK=64, rV=64, L_max=1024)
    a.update(kw)
    return lib.stief_compress_append(a["k"], a["v"], a["P_K"], a["P_V"], a["kl"], a["vl"],
                                     a["sl"], a["B"], a["Hkv"], a["T"], a["d"], a["rK"],
                                     a["rV"], a["L_max"], None, None)


@pytest.mark.parametrize("kw,code", [
    (dict(q=None), INVALID), (dict(out=None), INVALID), (dict(seq_lens=None), INVALID),
    (dict(d=64), INVALID), (dict(rK=8), INVALID), (dict(rV=72), INVALID), (dict(rK=144), INVALID),
    (dict(Hq=30), INVALID), (dict(B=0), INVALID), (dict(Hkv=0), INVALID),
    (dict(Hq=8 * 65, Hkv=8), INVALID), (dict(num_splits=-1), INVALID),
    (dict(num_splits=9), INVALID),  # max for 1024 tokens is 8
    (dict(max_seq_len=2048), CAPACITY), (dict(max_seq_len=-1), INVALID),
    (dict(q=FAKE + 8), ALIGN), (dict(k_lat=FAKE + 2), ALIGN), (dict(out=FAKE + 4), ALIGN),
    (dict(ws=None), WORKSPACE), (dict(ws_bytes=16), WORKSPACE),
])
def test_decode_argument_errors(lib, kw, code):
    assert _decode(lib, **kw) == code


def _latent(lib, **kw):
    a = dict(q=FAKE, k_lat=FAKE, v_lat=FAKE, seq_lens=FAKE, out=FAKE, ws=FAKE, ws_bytes=1 << 40,
             B=1, Hq=32, Hkv=8, d=128, rK=64, rV=48, L_max=1024, max_seq_len=1024, num_splits=0)
    a.update(kw)
    return lib.stief_decode_latent(a["q"], a["k_lat"], a["v_lat"], a["seq_lens"], a["out"],
                                   a["ws"], a["ws_bytes"], a["B"], a["Hq"], a["Hkv"], a["d"],
                                   a["rK"], a["rV"], a["L_max"], a["max_seq_len"],
                                   a["num_splits"], None, None)


@pytest.mark.parametrize("kw,code", [
    (dict(q=None), INVALID), (dict(k_lat=None), INVALID), (dict(out=None), INVALID),
    (dict(d=64), INVALID), (dict(rV=40), INVALID), (dict(Hq=30), INVALID),
    (dict(num_splits=9), INVALID), (dict(max_seq_len=2048), CAPACITY),
    (dict(q=FAKE + 8), ALIGN), (dict(v_lat=FAKE + 2), ALIGN), (dict(out=FAKE + 4), ALIGN),
    (dict(ws=None), WORKSPACE), (dict(ws_bytes=16), WORKSPACE),
])
def test_latent_decode_argument_errors(lib, kw, code):
    """The latent decode takes no bases: its checks are the decode's minus P_K / P_V."""
    assert _latent(lib, **kw) == code


def _joint(lib, latent=False, **kw):
    a = dict(q=FAKE, P_K=FAKE, P_VJ=FAKE, k_lat=FAKE, v_joint=FAKE, seq_lens=FAKE, out=FAKE,
             ws=FAKE, ws_bytes=1 << 40, B=1, Hq=32, Hkv=8, d=128, rK=64, rV=64, L_max=1024,
             max_seq_len=1024, num_splits=0)
    a.update(kw)
    tail = (a["ws"], a["ws_bytes"], a["B"], a["Hq"], a["Hkv"], a["d"], a["rK"], a["rV"],
            a["L_max"], a["max_seq_len"], a["num_splits"], None, None)
    if latent:
        return lib.stief_decode_latent_joint_v(a["q"], a["k_lat"], a["v_joint"], a["seq_lens"],
                                               a["out"], *tail)
    return lib.stief_decode_attention_joint_v(a["q"], a["P_K"], a["P_VJ"], a["k_lat"],
                                              a["v_joint"], a["seq_lens"], a["out"], *tail)


@pytest.mark.parametrize("latent", [False, True])
@pytest.mark.parametrize("kw,code", [
    (dict(q=None), INVALID), (dict(v_joint=None), INVALID), (dict(out=None), INVALID),
    (dict(d=64), INVALID), (dict(rV=40), INVALID), (dict(Hq=30), INVALID),
    (dict(max_seq_len=2048), CAPACITY), (dict(v_joint=FAKE + 2), ALIGN),
    (dict(ws_bytes=16), WORKSPACE),
])
def test_joint_value_decode_argument_errors(lib, latent, kw, code):
    """The joint-value calls check what the per-head decode and latent decode check."""
    assert _joint(lib, latent=latent, **kw) == code


@pytest.mark.parametrize("kw", [dict(P_K=None), dict(P_VJ=None)])
def test_joint_value_decode_needs_both_bases(lib, kw):
    assert _joint(lib, **kw) == INVALID


def _joint_compress(lib, **kw):
    a = dict(k=FAKE, v=FAKE, P_K=FAKE, P_VJ=FAKE, kl=FAKE, vj=FAKE, sl=FAKE, B=1, Hkv=8, T=1,
             d=128, rK=64, rV=64, L_max=1024)
    a.update(kw)
    return lib.stief_compress_append_joint_v(a["k"], a["v"], a["P_K"], a["P_VJ"], a["kl"],
                                             a["vj"], a["sl"], a["B"], a["Hkv"], a["T"], a["d"],
                                             a["rK"], a["rV"], a["L_max"], None, None)


@pytest.mark.parametrize("kw,code", [
    (dict(k=None), INVALID), (dict(P_VJ=None), INVALID), (dict(vj=None), INVALID),
    (dict(sl=None), INVALID), (dict(d=64), INVALID), (dict(rK=8), INVALID), (dict(rV=136), INVALID),
    (dict(B=0), INVALID), (dict(B=65536), INVALID), (dict(Hkv=0), INVALID), (dict(T=-1), INVALID),
    (dict(L_max=0), INVALID), (dict(T=2000), CAPACITY), (dict(vj=FAKE + 2), ALIGN),
    (dict(P_VJ=FAKE + 8), ALIGN), (dict(T=0), OK),
])
def test_joint_compress_argument_errors(lib, kw, code):
    """T = 0 is a no-op that returns OK without touching CUDA; everything else is refused
    before anything is launched."""
    assert _joint_compress(lib, **kw) == code


def _paged(lib, **kw):
    a = dict(q=FAKE, P_K=FAKE, P_V=FAKE, kp=FAKE, vp=FAKE, bt=FAKE, sl=FAKE, out=FAKE, ws=FAKE,
             ws_bytes=1 << 40, B=2, Hq=32, Hkv=8, d=128, rK=64, rV=64, num_pages=64,
             page_size=128, max_pages=16, max_seq_len=2048, num_splits=0)
    a.update(kw)
    return lib.stief_decode_attention_paged(a["q"], a["P_K"], a["P_V"], a["kp"], a["vp"], a["bt"],
                                            a["sl"], a["out"], a["ws"], a["ws_bytes"], a["B"],
                                            a["Hq"], a["Hkv"], a["d"], a["rK"], a["rV"],
                                            a["num_pages"], a["page_size"], a["max_pages"],
                                            a["max_seq_len"], a["num_splits"], None, None)


@pytest.mark.parametrize("kw,code", [
    (dict(bt=None), INVALID), (dict(page_size=96), INVALID), (dict(page_size=32), INVALID),
    (dict(num_pages=0), INVALID), (dict(max_pages=0), INVALID),
    (dict(max_seq_len=16 * 128 + 1), CAPACITY),  # beyond max_pages * page_size
    (dict(num_pages=1 << 20, page_size=1 << 12), INVALID),  # pool rows >= 2^31
    (dict(bt=FAKE + 2), ALIGN), (dict(kp=FAKE + 8), ALIGN), (dict(ws=None), WORKSPACE),
])
def test_paged_decode_argument_errors(lib, kw, code):
    """The paged decode checks the pool geometry and the block table before any CUDA call."""
    assert _paged(lib, **kw) == code


def _q8(lib, **kw):
    a = dict(q=FAKE, P_K=FAKE, P_V=FAKE, kq=FAKE, vq=FAKE, ks=FAKE, vs=FAKE, sl=FAKE, out=FAKE,
             ws=FAKE, ws_bytes=1 << 40, B=1, Hq=32, Hkv=8, d=128, rK=64, rV=64, L_max=1024,
             max_seq_len=1024, num_splits=0)
    a.update(kw)
    return lib.stief_decode_attention_q8(a["q"], a["P_K"], a["P_V"], a["kq"], a["vq"], a["ks"],
                                         a["vs"], a["sl"], a["out"], a["ws"], a["ws_bytes"], a["B"],
                                         a["Hq"], a["Hkv"], a["d"], a["rK"], a["rV"], a["L_max"],
                                         a["max_seq_len"], a["num_splits"], None, None)


@pytest.mark.parametrize("kw,code", [
    (dict(ks=None), INVALID), (dict(vs=None), INVALID),
    (dict(L_max=1000, max_seq_len=1000), INVALID),  # int8 caches: L_max a multiple of 64
    (dict(ks=FAKE + 4), ALIGN), (dict(kq=FAKE + 8), ALIGN), (dict(rK=40), INVALID),
    (dict(ws=None), WORKSPACE),
])
def test_q8_decode_argument_errors(lib, kw, code):
    assert _q8(lib, **kw) == code


def _q8_step(lib, **kw):
    a = dict(q=FAKE, kn=FAKE, vn=FAKE, P_K=FAKE, P_V=FAKE, kq=FAKE, vq=FAKE, ks=FAKE, vs=FAKE,
             sl=FAKE, out=FAKE, ws=FAKE, ws_bytes=1 << 40, B=1, Hq=32, Hkv=8, d=128, rK=64, rV=64,
             L_max=1024, max_seq_len=1024, num_splits=0)
    a.update(kw)
    return lib.stief_append_decode_q8(a["q"], a["kn"], a["vn"], a["P_K"], a["P_V"], a["kq"], a["vq"],
                                      a["ks"], a["vs"], a["sl"], a["out"], a["ws"], a["ws_bytes"],
                                      a["B"], a["Hq"], a["Hkv"], a["d"], a["rK"], a["rV"], a["L_max"],
                                      a["max_seq_len"], a["num_splits"], None, None)


@pytest.mark.parametrize("kw,code", [
    (dict(kn=None), INVALID), (dict(vn=None), INVALID), (dict(ks=None), INVALID),
    (dict(L_max=1000, max_seq_len=1000), INVALID), (dict(vn=FAKE + 2), ALIGN),
    (dict(vs=FAKE + 4), ALIGN), (dict(max_seq_len=2048), CAPACITY), (dict(ws=None), WORKSPACE),
])
def test_q8_fused_step_argument_errors(lib, kw, code):
    """The int8 fused step checks its new rows, scales and cache geometry before any CUDA
    call."""
    assert _q8_step(lib, **kw) == code


@pytest.mark.parametrize("kw,code", [
    (dict(k=None), INVALID), (dict(sl=None), INVALID), (dict(d=96), INVALID),
    (dict(rK=24), INVALID), (dict(T=-1), INVALID), (dict(B=0), INVALID),
    (dict(T=2048), CAPACITY), (dict(kl=FAKE + 4), ALIGN), (dict(P_V=FAKE + 8), ALIGN),
    (dict(T=0), OK),  # nothing to do: returns before any CUDA call
])
def test_compress_argument_errors(lib, kw, code):
    assert _compress(lib, **kw) == code


def test_split_planning():
    assert stief.stief_decode_max_splits(0) == 1
    assert stief.stief_decode_max_splits(128) == 1
    assert stief.stief_decode_max_splits(129) == 2
    assert stief.stief_decode_max_splits(10 ** 9) == 512
    assert stief.stief_decode_max_splits(-1) == 0
    # one split CTA per SM: 8 KV heads at batch 1 on 148 SMs -> 18 splits
    assert stief.stief_decode_auto_splits(1, 32, 8, 32768, 148) == 18
    assert stief.stief_decode_auto_splits(1, 32, 8, 131072, 148) == 18
    assert stief.stief_decode_auto_splits(1, 4, 1, 1024, 148) == 8     # capped by the length
    assert stief.stief_decode_auto_splits(16, 32, 8, 8192, 148) == 1
    assert stief.stief_decode_auto_splits(64, 32, 8, 4096, 148) == 1
    assert stief.stief_decode_auto_splits(1, 64, 2, 32768, 148) == 18   # G=32 -> 4 sub-groups
    assert stief.stief_decode_auto_splits(1, 16, 1, 32768, 148) == 74   # G=16 -> 2 sub-groups
    for B in (1, 2, 5, 64):
        for L in (1, 100, 5000, 200000):
            s = stief.stief_decode_auto_splits(B, 32, 8, L, 148)
            assert 1 <= s <= stief.stief_decode_max_splits(L)
            assert s == 1 or B * 8 * s <= 148


def test_workspace_bytes():
    # (units + B) uint32 ticket counters padded to 256 bytes, then [units * G_T * max_splits]
    # partial-state records of (d + 2) 8-byte words: a tagged record holds o~[r_V], m and l
    # as (value, tag) words, a ticket record r_V + 4 floats (the value rank does not change
    # the size)
    assert stief.stief_decode_workspace_bytes(1, 32, 8, 64, 32768) == 256 + 8 * 4 * 256 * 130 * 8
    assert stief.stief_decode_workspace_bytes(2, 24, 8, 48, 100) == 256 + 16 * 4 * 1 * 130 * 8
    assert stief.stief_decode_workspace_bytes(64, 32, 8, 64, 4096) == 2304 + 512 * 4 * 32 * 130 * 8
    assert stief.stief_decode_workspace_bytes(1, 32, 8, 72, 100) == 0
    assert stief.stief_decode_workspace_bytes(1, 30, 8, 64, 100) == 0


def test_prepare_validates_like_the_call():
    """stief.prepare runs the binding function's own checks (no launch): a CPU tensor is
    refused with the same error as the direct call, and the capture state is cleared after."""
    import torch
    import decode_attention_stief_b200 as stief
    from decode_attention_stief_b200 import _binding
    q = torch.zeros(1, 4, 128, dtype=torch.bfloat16)
    with pytest.raises(ValueError, match="q must be on a CUDA device"):
        stief.prepare(stief.stief_decode_attention, q, None, None, None, None, None, None, None, 0)
    assert getattr(_binding._capture, "calls", None) is None
