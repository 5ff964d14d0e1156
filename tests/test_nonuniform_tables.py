"""The library's host tables of the non-uniform angle quantiser
(spkv_nonuniform_tables: quadrature of sin^k and Newton inversion) against the
oracle's quantiles (oracle/nonuniform.py: the regularised incomplete beta
function and its inverse).  CPU only: the tables are built on the host."""
import math

import numpy as np
import pytest

from oracle import nonuniform as nu


@pytest.fixture(scope="module")
def ops():
    from compressed_kv_decode_ada_b200 import ops

    return ops


@pytest.mark.parametrize("d,b", [(3, 2), (3, 4), (16, 3), (128, 3), (128, 4), (128, 8)])
def test_tables_match_the_oracle_quantiles(ops, d, b):
    ec, mc, ms = ops.nonuniform_tables(d, b)
    np.testing.assert_allclose(ec, np.cos(nu.polar_edges(d, b)), rtol=0, atol=1e-12)
    mids = nu.polar_mids(d, b)
    np.testing.assert_allclose(mc, np.cos(mids), rtol=0, atol=1e-12)
    np.testing.assert_allclose(ms, np.sin(mids), rtol=0, atol=1e-12)


def test_d3_closed_form(ops):
    """d = 3: cos(edge j) = 1 - 2 j / 2^b and cos(median j) = 1 - (2 j + 1) / 2^b."""
    ec, mc, _ = ops.nonuniform_tables(3, 5)
    n = 32
    np.testing.assert_allclose(ec[0], 1 - 2 * np.arange(1, n) / n, atol=1e-13)
    np.testing.assert_allclose(mc[0], 1 - (2 * np.arange(n) + 1) / n, atol=1e-13)


def test_arguments_are_checked(ops):
    from compressed_kv_decode_ada_b200._lib import SpkvError

    for d, b in ((2, 3), (128, 0), (128, 13)):
        with pytest.raises(SpkvError):
            ops.nonuniform_tables(d, b)
    assert math.isfinite(float(ops.nonuniform_tables(4, 1)[1][0, 0]))
