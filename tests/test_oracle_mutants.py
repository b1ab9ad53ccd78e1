"""Plant a mistake in a copy of the oracle's C source; some pin must catch it.

Each mutant is a plausible slip (wrong scale, wrong GQA mapping, transposed
basis, missing normalisation, off-by-one in the append offset, ...).  The copy is
compiled with gcc into a temporary directory and exercised in a child process
(an off-by-one may write outside an array, so the child may also die: that
counts as caught).  The oracle source itself is never changed.
"""
import json
import os
import subprocess
import sys

import numpy as np
import pytest

import oracle

SRC = os.path.join(os.path.dirname(oracle.__file__), "stief_oracle.c")
TESTS = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(TESTS)

# (name, original text, replacement, checks expected to fail)
MUTANTS = [
    ("scale_uses_rank", "1.0 / sqrt((double)d)", "1.0 / sqrt((double)rK)",
     ["two_tokens", "tiny_compressed_is_sdpa_on_reconstructed_rows"]),
    ("gqa_interleaved", "(long)g * G + j", "(long)j * Hkv + g",
     ["full_rank_is_plain_attention", "tiny_compressed_is_sdpa_on_reconstructed_rows"]),
    ("reconstruct_transposed", "acc += lat[c] * P[(long)i * r + c];",
     "acc += lat[c] * P[(long)c * d + i];",
     ["single_token", "gauge_invariance", "tiny_compressed_is_sdpa_on_reconstructed_rows"]),
    ("compress_transposed", "acc += x[t * d + i] * P[(long)i * r + c];",
     "acc += x[t * d + i] * P[(long)c * d + i];",
     ["compress_identity_basis", "full_rank_is_plain_attention"]),
    ("no_max_subtraction", "sj[t] = exp(sj[t] - mx);", "sj[t] = exp(sj[t]);",
     ["full_rank_large_scores"]),
    ("unnormalised_weights", "double p = s[(long)j * L + t] / denom[j];",
     "double p = s[(long)j * L + t];",
     ["two_tokens", "uniform_keys", "tiny_compressed_is_sdpa_on_reconstructed_rows"]),
    ("values_use_key_basis", "reconstruct_row(Vd + t * rV, PV, d, rV, row);",
     "reconstruct_row(Vd + t * rV, PK, d, rV, row);",
     ["full_rank_is_plain_attention", "tiny_compressed_is_sdpa_on_reconstructed_rows"]),
    ("first_value_dropped",
     "for (long t = 0; t < L; ++t) {\n            reconstruct_row(Vd",
     "for (long t = 1; t < L; ++t) {\n            reconstruct_row(Vd",
     ["single_token", "two_tokens", "tiny_compressed_is_sdpa_on_reconstructed_rows"]),
    ("latent_scale_uses_rank", "w_lat[t] = acc * inv_sqrt_d;",
     "w_lat[t] = acc / sqrt((double)rK);", ["latent_is_sdpa_on_latent_rows"]),
    ("latent_gqa_interleaved", "const long head = (long)b * Hq + (long)g * G + j;",
     "const long head = (long)b * Hq + (long)j * Hkv + g;",
     ["latent_is_sdpa_on_latent_rows", "latent_folding_identity"]),
    ("latent_unnormalised", "const double p_lat = w_lat[t] / sum_lat;",
     "const double p_lat = w_lat[t];", ["latent_is_sdpa_on_latent_rows"]),
    ("latent_no_max_subtraction", "w_lat[t] = exp(w_lat[t] - mx);", "w_lat[t] = exp(w_lat[t]);",
     ["latent_large_scores"]),
    ("latent_values_from_keys", "oh[c] += p_lat * Vd[t * rV + c];",
     "oh[c] += p_lat * Kd[t * rK + c];", ["latent_is_sdpa_on_latent_rows", "latent_edges"]),
    ("round_ties_away", "nearbyint(x / q)", "round(x / q)",
     ["round_bf16_edges", "round_bf16_matches_torch"]),
    ("append_off_by_one", "long dst = ((long)b * Hkv + h) * L_max + L;",
     "long dst = ((long)b * Hkv + h) * L_max + L + 1;", ["compress_append_bookkeeping"]),
    ("capacity_rejects_exact_fit", "if (L < 0 || L + T > L_max) {",
     "if (L < 0 || L + T >= L_max) {", ["compress_append_bookkeeping"]),
]

_CHILD = r"""
import json, sys
sys.path[:0] = [{root!r}, {tests!r}]
import oracle, oracle_checks as oc
m = oracle.Oracle({lib!r})
caught = {{}}
for name in {checks!r}:
    try:
        oc.ALL_ORACLE_CHECKS[name](m)
        caught[name] = False
    except (AssertionError, ValueError):
        caught[name] = True
print(json.dumps(caught))
"""


@pytest.mark.parametrize("name,orig,repl,checks", MUTANTS, ids=[m[0] for m in MUTANTS])
def test_mutant_is_caught(tmp_path, name, orig, repl, checks):
    src = open(SRC).read()
    assert src.count(orig) >= 1, f"mutation site for {name} not found"
    mutated = tmp_path / f"{name}.c"
    mutated.write_text(src.replace(orig, repl))
    lib = oracle.build(str(mutated), str(tmp_path / f"{name}.so"), force=True)
    code = _CHILD.format(root=ROOT, tests=TESTS, lib=lib, checks=checks)
    proc = subprocess.run([sys.executable, "-c", code], capture_output=True, text=True,
                          timeout=300)
    if proc.returncode != 0:
        return  # the planted mistake crashed the child (e.g. an out-of-bounds write): caught
    caught = json.loads(proc.stdout.strip().splitlines()[-1])
    missed = [c for c, ok in caught.items() if not ok]
    assert not missed, f"mutant {name} passed pins {missed}"


# The joint-value calls are layout (concatenation order, the block of P_VJ each KV head reads,
# the value latent every head shares) over the C functions above.  Their planted mistakes are
# subclasses that override one layout helper; they touch no memory, so they run in-process.

def _interleaved_concat(x):
    Hkv, T, d = x.shape
    return np.ascontiguousarray(np.transpose(x, (1, 2, 0)).reshape(T, d * Hkv))


def _interleaved_blocks(P_VJ, Hkv):
    HD, rV = P_VJ.shape
    return np.ascontiguousarray(np.transpose(P_VJ.reshape(HD // Hkv, Hkv, rV), (1, 0, 2)))


def _block0_everywhere(P_VJ, Hkv):
    HD, rV = P_VJ.shape
    return np.ascontiguousarray(np.broadcast_to(P_VJ[:HD // Hkv][None], (Hkv, HD // Hkv, rV)))


def _values_for_head0_only(v_joint, Hkv):
    B, L, rV = v_joint.shape
    out = np.zeros((B, Hkv, L, rV))
    out[:, 0] = v_joint
    return out


JOINT_MUTANTS = [
    ("joint_concat_interleaved", "_concat_heads", _interleaved_concat,
     ["joint_v_full_rank_is_plain_attention", "joint_v_block_diagonal_is_per_head",
      "joint_v_compress_bookkeeping"]),
    ("joint_blocks_interleaved", "_head_blocks", _interleaved_blocks,
     ["joint_v_full_rank_is_plain_attention", "joint_v_block_diagonal_is_per_head",
      "joint_v_edges"]),
    ("joint_every_head_reads_block0", "_head_blocks", _block0_everywhere,
     ["joint_v_full_rank_is_plain_attention", "joint_v_block_diagonal_is_per_head",
      "joint_v_edges"]),
    ("joint_values_for_head0_only", "_share_values", _values_for_head0_only,
     ["joint_v_full_rank_is_plain_attention", "joint_v_edges"]),
]


@pytest.mark.parametrize("name,helper,wrong,checks", JOINT_MUTANTS, ids=[m[0] for m in JOINT_MUTANTS])
def test_joint_mutant_is_caught(name, helper, wrong, checks):
    import oracle_checks as oc
    mutant_cls = type("Mutant", (oracle.Oracle,), {helper: staticmethod(wrong)})
    m = mutant_cls(oracle.build())
    missed = []
    for c in checks:
        try:
            oc.ALL_ORACLE_CHECKS[c](m)
            missed.append(c)
        except (AssertionError, ValueError):
            pass
    assert not missed, f"mutant {name} passed pins {missed}"
