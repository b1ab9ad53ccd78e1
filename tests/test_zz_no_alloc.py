"""stief_decode_attention_noalloc: the decode entry point for callers that cannot allocate.

Some callers cannot allocate device memory where they decode: a serving engine whose
KV-cache pool already holds nearly all of HBM, an operator interface that passes only
inputs and outputs, or a loop that must not call cudaMalloc.  This entry point keeps its
split partial states in a fixed device array owned by the library instead of a caller
workspace.  These tests call it through the C ABI and check its output against
stief_decode_attention (the workspace entry point) and against the fp64 oracle, within the
parity tolerance, on two calls in a row with different inputs, and that sizes beyond its
fixed scratch are refused before anything is launched.  They pass alone in a fresh process
as well as after the other GPU files.
"""
import ctypes

import pytest
import torch

import decode_attention_stief_b200 as stief
from gpu_util import DECODE_TOL, decode_error, f64, make_decode_case, oracle_decode

pytestmark = pytest.mark.gpu


def _both(case, lens, max_seq_len):
    dev = torch.device("cuda")
    q, P_K, P_V, k_lat, v_lat = (x.to(dev) for x in case)
    lens_t = torch.tensor(lens, dtype=torch.int32, device=dev)
    B, Hq, d = q.shape
    ref = torch.empty((B, Hq, d), dtype=torch.bfloat16, device=dev)
    ws = stief.workspace_for(B, Hq, P_K.shape[0], P_V.shape[2], max_seq_len)
    stief.stief_decode_attention(q, P_K, P_V, k_lat, v_lat, lens_t, ref, ws, max_seq_len)
    got = torch.full((B, Hq, d), float("nan"), dtype=torch.bfloat16, device=dev)
    status = torch.zeros(1, dtype=torch.int32, device=dev)
    stief.stief_decode_attention_noalloc(q, P_K, P_V, k_lat, v_lat, lens_t, got, max_seq_len,
                                         dev_status=status)
    assert stief.stief_read_device_status(status) == 0
    return got.cpu(), ref.cpu()


def test_noalloc_matches_workspace_entry_point_two_calls():
    # first call: GQA 4, ranks 64/48, ragged lengths with several splits
    case1 = make_decode_case(2, 32, 8, 64, 48, 3000, 4242)
    got1, ref1 = _both(case1, [3000, 1777], 3000)
    assert decode_error(got1, f64(ref1)) <= DECODE_TOL
    assert decode_error(got1, oracle_decode(*case1, [3000, 1777])) <= DECODE_TOL
    # second call right after, different sizes: the scratch holds the first call's data
    case2 = make_decode_case(3, 16, 2, 32, 96, 700, 4343)
    got2, ref2 = _both(case2, [700, 0, 129], 700)
    assert decode_error(got2, f64(ref2)) <= DECODE_TOL
    assert decode_error(got2, oracle_decode(*case2, [700, 0, 129])) <= DECODE_TOL
    assert torch.all(got2[1].float() == 0)


def test_noalloc_refuses_sizes_beyond_its_scratch():
    lib = stief.library()
    fake = 0x10000  # aligned, never dereferenced: the call returns before launching
    # 1024 sequences x 32 query heads x (128 + 2) floats > 8 MiB
    code = lib.stief_decode_attention_noalloc(fake, fake, fake, fake, fake, fake, fake, 1024, 32,
                                              8, 128, 64, 128, 4096, 4096, 0, None, None)
    assert code == 4, stief.stief_status_string(code)  # STIEF_ERR_WORKSPACE
