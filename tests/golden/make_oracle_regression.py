"""Write oracle_regression.json: the oracle's results on a few small seeded cases.

The pages print no worked numerical example of the method (the StiefAttention summaries give
its algebra and quality tables, no input/output pair), so no fixture in this folder holds a
value taken from them.  This record freezes what the pinned oracle computes, so that a later
change to its arithmetic shows up as a diff of this file and has to say which passage, or
which reading of it, justifies the change.  It calls only ``oracle`` and the seeded input
generators; regenerate with ``python tests/golden/make_oracle_regression.py``.
"""
from __future__ import annotations

import hashlib
import json
import os
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(os.path.dirname(HERE))
sys.path[:0] = [ROOT]

import numpy as np  # noqa: E402

import oracle  # noqa: E402
import stief_inputs as si  # noqa: E402

OUT = os.path.join(HERE, "oracle_regression.json")

# small shapes: GQA groups of 2; decode over a full, a ragged and an empty sequence
B, Hq, Hkv, d, rK, rV, T, L_max = 3, 4, 2, 32, 16, 8, 20, 24
LENS0 = [0, 0, 0]            # lengths before the append
DECODE_LENS = [20, 13, 0]    # lengths the decode attends to: full, ragged, empty
SEED = 4242


def inputs():
    """The seeded inputs of every case (bf16 values held as fp64)."""
    k_new, v_new = si.full_kv(SEED, B, Hkv, T, d)
    P_K, P_V = si.bases_bf16(SEED, Hkv, d, rK, rV)
    P_VJ = si.to_bf16(si.bases(SEED + 2, 1, Hkv * d, 2 * rV)[0])
    q = si.queries(SEED, B, Hq, d)
    f = si.bf16_to_f64
    return {"k_new": f(k_new), "v_new": f(v_new), "P_K": f(P_K), "P_V": f(P_V),
            "P_VJ": f(P_VJ), "q": f(q)}


def results(o=None):
    """Every recorded array, computed by the oracle ``o`` (the default one if None)."""
    o = o or oracle.default()
    x = inputs()
    lens0 = np.array(LENS0, np.int32)
    k_lat, v_lat, lens, nbad = o.compress_append(
        x["k_new"], x["v_new"], x["P_K"], x["P_V"], np.zeros((B, Hkv, L_max, rK)),
        np.zeros((B, Hkv, L_max, rV)), lens0)
    dl = np.array(DECODE_LENS, np.int32)
    out = o.decode(x["q"], x["P_K"], x["P_V"], k_lat, v_lat, dl)
    G = Hq // Hkv
    q_lat = np.stack([np.stack([x["q"][b, h] @ x["P_K"][h // G] for h in range(Hq)])
                      for b in range(B)])
    out_lat = o.decode_latent(q_lat, k_lat, v_lat, dl, d=d)
    kj, vj, lj, nbj = o.compress_append_joint_v(
        x["k_new"], x["v_new"], x["P_K"], x["P_VJ"], np.zeros((B, Hkv, L_max, rK)),
        np.zeros((B, L_max, 2 * rV)), lens0)
    out_j = o.decode_joint_v(x["q"], x["P_K"], x["P_VJ"], kj, vj, dl)
    codes, scales = oracle.quantize_rows(k_lat)  # the int8 form of the key cache
    return {
        "compress_k_lat": k_lat, "compress_v_lat": v_lat,
        "compress_lens": lens.astype(np.float64), "compress_overflow": np.array([float(nbad)]),
        "decode_out": out, "decode_latent_out": out_lat,
        "joint_v_cache": vj, "joint_v_lens": lj.astype(np.float64),
        "joint_v_overflow": np.array([float(nbj)]), "decode_joint_v_out": out_j,
        "int8_codes": codes.astype(np.float64), "int8_scales": scales.astype(np.float64),
    }


def sha(a: np.ndarray) -> str:
    return hashlib.sha256(np.ascontiguousarray(a, np.float64).tobytes()).hexdigest()


def main():
    rec = {
        "_what": "oracle results on small seeded cases (not page values: the pages print none)",
        "_script": "tests/golden/make_oracle_regression.py",
        "shapes": {"B": B, "Hq": Hq, "Hkv": Hkv, "d": d, "rK": rK, "rV": rV, "T": T,
                   "L_max": L_max, "lens_before_append": LENS0, "decode_lens": DECODE_LENS,
                   "seed": SEED},
        "arrays": {},
    }
    for name, a in results().items():
        entry = {"shape": list(a.shape), "sha256": sha(a)}
        if name.endswith("_out"):
            entry["hex"] = [float(v).hex() for v in a.ravel()]
        rec["arrays"][name] = entry
    with open(OUT, "w") as fh:
        json.dump(rec, fh, indent=0)
        fh.write("\n")
    print(f"wrote {OUT}")


if __name__ == "__main__":
    main()
