"""Change of coordinates inside the subspace on the GPU (StiefAttention technical summary,
"Mecanismo Central" item 3: the QR factor R only changes coordinates).  With P -> P.O for an
orthogonal r x r matrix O (a random rotation, and a column sign flip), compressing the same
full keys and values and decoding gives the same output within the decode tolerance: the
latent rows change, what the attention sees does not.  Each output is also checked against the
oracle on its own bases."""
import numpy as np
import pytest
import torch

import decode_attention_stief_b200 as stief
import oracle
import stief_inputs as si
from gpu_util import DECODE_TOL, assert_decode_close, decode_error, f64

pytestmark = pytest.mark.gpu
DEV = torch.device("cuda")


def _compress_decode(k_new, v_new, q, P_K, P_V, L_max):
    B, Hkv, T, d = k_new.shape
    Hq = q.shape[1]
    rK, rV = P_K.shape[2], P_V.shape[2]
    k_lat = torch.zeros((B, Hkv, L_max, rK), dtype=torch.bfloat16, device=DEV)
    v_lat = torch.zeros((B, Hkv, L_max, rV), dtype=torch.bfloat16, device=DEV)
    lens = torch.zeros(B, dtype=torch.int32, device=DEV)
    status = torch.zeros(1, dtype=torch.int32, device=DEV)
    stief.stief_compress_append(k_new.to(DEV), v_new.to(DEV), P_K.to(DEV), P_V.to(DEV), k_lat,
                                v_lat, lens, dev_status=status)
    out = torch.empty((B, Hq, d), dtype=torch.bfloat16, device=DEV)
    ws = stief.workspace_for(B, Hq, Hkv, rV, L_max)
    stief.stief_decode_attention(q.to(DEV), P_K.to(DEV), P_V.to(DEV), k_lat, v_lat, lens, out,
                                 ws, L_max, dev_status=status)
    assert stief.stief_read_device_status(status) == 0
    return out.cpu()


def _oracle(k_new, v_new, q, P_K, P_V, L_max):
    B, Hkv, T, d = k_new.shape
    rK, rV = P_K.shape[2], P_V.shape[2]
    kl, vl, lens, _ = oracle.compress_append(f64(k_new), f64(v_new), f64(P_K), f64(P_V),
                                             np.zeros((B, Hkv, L_max, rK)),
                                             np.zeros((B, Hkv, L_max, rV)), np.zeros(B, np.int32))
    return oracle.decode(f64(q), f64(P_K), f64(P_V), kl, vl, lens)


@pytest.mark.parametrize("kind", ["rotation", "sign_flip"])
def test_basis_change_leaves_the_output(kind):
    B, Hq, Hkv, d, rK, rV, T = 2, 16, 4, 128, 64, 48, 200
    k_new, v_new = si.full_kv(8300, B, Hkv, T, d)
    q = si.queries(8300, B, Hq, d)
    PK = si.bases(8301, Hkv, d, rK)
    PV = si.bases(8302, Hkv, d, rV)
    rng = np.random.default_rng(8303)
    if kind == "rotation":
        OK = np.stack([si.stiefel_basis(rng, rK, rK) for _ in range(Hkv)])
        OV = np.stack([si.stiefel_basis(rng, rV, rV) for _ in range(Hkv)])
    else:
        OK = np.stack([np.diag(rng.choice([-1.0, 1.0], rK)) for _ in range(Hkv)])
        OV = np.stack([np.diag(rng.choice([-1.0, 1.0], rV)) for _ in range(Hkv)])
    outs = []
    for P_K, P_V in ((PK, PV), (PK @ OK, PV @ OV)):
        P_K, P_V = si.to_bf16(P_K), si.to_bf16(P_V)
        got = _compress_decode(k_new, v_new, q, P_K, P_V, T)
        assert_decode_close(got, _oracle(k_new, v_new, q, P_K, P_V, T))
        outs.append(got)
    err = decode_error(outs[1], f64(outs[0]))
    assert err <= DECODE_TOL, f"basis change moved the output by {err:.3e} of ||o||_inf"
