"""Helpers for the GPU parity tests: run the CUDA path through the C-ABI binding
and the fp64 oracle on the same seeded inputs, and compare."""
from __future__ import annotations

import numpy as np
import torch

import decode_attention_stief_b200 as stief
import oracle
import stief_inputs as si

# spec tolerance for bf16 storage with fp32 accumulation
DECODE_TOL = 2e-2


def f64(t: torch.Tensor) -> np.ndarray:
    return t.detach().to("cpu", torch.float64).numpy()


_ws_cache = {}


def _workspace(B, Hq, Hkv, rV, max_seq_len):
    """One zero-filled workspace per size, reused across calls (its counters stay zero)."""
    key = (B, Hq, Hkv, rV, max_seq_len)
    if key not in _ws_cache:
        _ws_cache[key] = stief.workspace_for(*key)
    return _ws_cache[key]


def gpu_decode(q, P_K, P_V, k_lat, v_lat, lens, num_splits=0, max_seq_len=None,
               expect_status=0) -> torch.Tensor:
    """Decode on the GPU through stief_decode_attention; inputs may live on CPU or GPU."""
    dev = torch.device("cuda")
    q, P_K, P_V, k_lat, v_lat = (x.to(dev).contiguous() for x in (q, P_K, P_V, k_lat, v_lat))
    lens_t = torch.as_tensor(np.asarray(lens, dtype=np.int32)).to(dev)
    B, Hq, d = q.shape
    Hkv = P_K.shape[0]
    rV = P_V.shape[2]
    if max_seq_len is None:
        max_seq_len = int(np.max(np.asarray(lens))) if len(lens) else 0
    out = torch.full((B, Hq, d), float("nan"), dtype=torch.bfloat16, device=dev)
    ws = _workspace(B, Hq, Hkv, rV, max_seq_len)
    status = torch.zeros(1, dtype=torch.int32, device=dev)
    stief.stief_decode_attention(q, P_K, P_V, k_lat, v_lat, lens_t, out, ws, max_seq_len,
                                 num_splits=num_splits, dev_status=status)
    st = stief.stief_read_device_status(status)
    assert st == expect_status, f"device status {st:#x}"
    return out.cpu()


def oracle_decode(q, P_K, P_V, k_lat, v_lat, lens) -> np.ndarray:
    return oracle.decode(f64(q), f64(P_K), f64(P_V), f64(k_lat), f64(v_lat),
                         np.asarray(lens, dtype=np.int32))


def decode_error(got: torch.Tensor, want: np.ndarray) -> float:
    """max |got - want| / max |want| (want == 0 everywhere -> absolute error)."""
    g = f64(got)
    assert np.all(np.isfinite(g)), "non-finite output"
    scale = float(np.max(np.abs(want)))
    err = float(np.max(np.abs(g - want)))
    return err / scale if scale > 0 else err


def assert_decode_close(got, want, tol=DECODE_TOL):
    err = decode_error(got, want)
    assert err <= tol, f"max|err| / ||o||_inf = {err:.3e} > {tol}"
    return err


def bf16_ulp(x: np.ndarray) -> np.ndarray:
    """Spacing of bf16 values at |x| (normal range)."""
    ax = np.maximum(np.abs(x), 2.0 ** -126)
    return np.exp2(np.floor(np.log2(ax)) - 7)


def make_decode_case(B, Hq, Hkv, rK, rV, L_max, seed, d=128, q_scale=1.0):
    """Seeded decode inputs (CPU bf16): q, P_K, P_V, k_lat, v_lat."""
    q = si.queries(seed, B, Hq, d, scale=q_scale)
    P_K, P_V = si.bases_bf16(seed, Hkv, d, rK, rV)
    k_lat = si.latent_cache(seed, B, Hkv, L_max, rK, 0)
    v_lat = si.latent_cache(seed, B, Hkv, L_max, rV, 1)
    return q, P_K, P_V, k_lat, v_lat
