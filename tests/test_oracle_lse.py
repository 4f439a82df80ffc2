"""Pins for the oracle's row statistics (log-sum-exp, argmax, top-k): closed
forms and an independent library routine, never the oracle's own formula."""
import math

import numpy as np
import pytest
from scipy.special import logsumexp

from svtest_util import bf16_bits, bf16_to_f32

pytestmark = pytest.mark.filterwarnings("ignore::RuntimeWarning")


def rows(values):
    v = np.asarray(values, dtype=np.float32)
    return [v, bf16_bits(v)]


@pytest.mark.parametrize("V", [1, 2, 7, 1024, 128256])
@pytest.mark.parametrize("T", [1.0, 0.7, 2.5])
def test_lse_constant_row_closed_form(svo, V, T):
    # every entry c: ln(V e^{c/T}) = c/T + ln V
    c = 1.375
    for row in rows(np.full(V, c)):
        expect = c / T + math.log(V)
        assert abs(svo.row_lse(row, T) - expect) <= 1e-12 * max(1.0, abs(expect))


@pytest.mark.parametrize("n1,n2,a,b,T", [(1, 1, 0.0, 1.0, 1.0), (3, 5, -2.5, 4.0, 0.7),
                                         (100, 1, 0.0, 12.0, 1.0), (7, 9000, 3.0, -3.0, 2.0)])
def test_lse_two_valued_row_closed_form(svo, n1, n2, a, b, T):
    # n1 entries a and n2 entries b: a/T + ln(n1 + n2 e^{(b-a)/T})
    vals = np.array([a] * n1 + [b] * n2, dtype=np.float32)
    np.random.default_rng(1).shuffle(vals)
    expect = a / T + math.log(n1 + n2 * math.exp((b - a) / T))
    for row in rows(vals):
        assert abs(svo.row_lse(row, T) - expect) <= 1e-12 * max(1.0, abs(expect))


def test_lse_masked_entries_drop_out(svo):
    # -inf masks a token: the LSE is that of the remaining entries
    vals = np.full(50, 0.5, dtype=np.float32)
    vals[::3] = -np.inf
    n = int(np.isfinite(vals).sum())
    for row in rows(vals):
        assert abs(svo.row_lse(row, 1.0) - (0.5 + math.log(n))) < 1e-12
    for row in rows(np.full(9, -np.inf)):
        assert svo.row_lse(row, 1.0) == -math.inf


@pytest.mark.parametrize("T", [1.0, 0.7])
def test_lse_matches_scipy_on_random_rows(svo, T):
    rng = np.random.default_rng(7)
    for V in (5, 1000, 128256):
        z = (rng.standard_normal(V) * 3).astype(np.float32)
        f32, bits = rows(z)
        ref32 = logsumexp(z.astype(np.float64) / T)
        ref16 = logsumexp(bf16_to_f32(bits).astype(np.float64) / T)
        assert abs(svo.row_lse(f32, T) - ref32) <= 1e-12 * abs(ref32)
        assert abs(svo.row_lse(bits, T) - ref16) <= 1e-12 * abs(ref16)


def test_lse_large_offsets_do_not_overflow(svo):
    # shifting a row by c shifts its LSE by c/T; huge logits must not overflow
    rng = np.random.default_rng(3)
    z = rng.standard_normal(333).astype(np.float32)
    zs = (z + np.float32(1.0e4)).astype(np.float32)
    shifted = svo.row_lse(zs, 0.5)
    ref = logsumexp(zs.astype(np.float64) / 0.5)
    assert math.isfinite(shifted)
    assert abs(shifted - ref) <= 1e-13 * abs(ref)
    # a constant +1e4 on every entry of a constant row: exactly c/T + ln V
    assert abs(svo.row_lse(np.full(333, 1.0e4, np.float32), 0.5)
               - (2.0e4 + math.log(333))) <= 1e-12 * 2.0e4


def test_argmax_lowest_index_on_ties_brute_force(svo):
    rng = np.random.default_rng(11)
    for V in (1, 2, 8, 300, 4099):
        for _ in range(20):
            # quantised values make ties common (as in bf16 logits)
            z = np.round(rng.standard_normal(V) * 2).astype(np.float32)
            for row in rows(z):
                assert svo.row_argmax(row) == int(np.argmax(z))


def test_argmax_with_masked_and_negative(svo):
    z = np.full(10, -np.inf, dtype=np.float32)
    z[7] = -1e30
    z[3] = -1e30
    assert svo.row_argmax(z) == 3
