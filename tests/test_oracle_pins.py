"""The fp64 oracle against its pins (CPU only).

See ``oracle_checks.py`` for what each check ties the oracle to.
"""
import pytest

import oracle
import oracle_checks as oc


@pytest.fixture(scope="module")
def orc():
    return oracle.default()


@pytest.mark.parametrize("name", sorted(oc.ALL_ORACLE_CHECKS))
def test_oracle_pin(orc, name):
    oc.ALL_ORACLE_CHECKS[name](orc)


def test_qr_bases_orthonormal():
    oc.check_qr_bases_orthonormal()


def test_oracle_thread_count_does_not_change_bits(orc):
    """OpenMP runs independent (sequence, KV head) problems; results are bitwise equal."""
    import numpy as np
    import stief_inputs as si
    rng = np.random.default_rng(3)
    B, Hq, Hkv, L, r, d = 3, 8, 2, 50, 32, 128
    q = rng.standard_normal((B, Hq, d))
    P = si.bases(5, Hkv, d, r)
    k = rng.standard_normal((B, Hkv, L, r))
    v = rng.standard_normal((B, Hkv, L, r))
    lens = np.array([50, 7, 0], np.int32)
    a = orc.decode(q, P, P, k, v, lens, num_threads=1)
    b = orc.decode(q, P, P, k, v, lens, num_threads=4)
    assert np.array_equal(a, b)
