"""Pins of the oracle's Hadamard matrix and fp32 butterfly rotation.

"Sage v2 improvements": the Hadamard matrix is built once and reused. The
pins are the defining identities (H H^T = D I, symmetry, +-1 entries), the
library routine scipy.linalg.hadamard (same Sylvester ordering), exact
agreement of the butterfly with x @ H on small integers, the involution
fwht(fwht(x)) = D x, and an fp32 error bound on random data."""
import math

import numpy as np
import pytest
import scipy.linalg

DS = [1, 2, 4, 8, 16, 32, 64, 128, 256]


@pytest.mark.parametrize("D", DS)
def test_hadamard_identity_and_symmetry(oracle_mod, D):
    H = oracle_mod.hadamard(D).astype(np.int64)
    assert set(np.unique(H)) <= {-1, 1}
    assert np.array_equal(H, H.T)
    assert np.array_equal(H @ H.T, D * np.eye(D, dtype=np.int64))


@pytest.mark.parametrize("D", DS)
def test_hadamard_matches_scipy(oracle_mod, D):
    assert np.array_equal(oracle_mod.hadamard(D), scipy.linalg.hadamard(D))


def test_hadamard_rejects_non_power_of_two(oracle_mod):
    with pytest.raises(ValueError):
        oracle_mod.hadamard(96)


@pytest.mark.parametrize("D", [64, 128])
def test_fwht_exact_on_small_integers(oracle_mod, D):
    rng = np.random.default_rng(D)
    x = rng.integers(-1000, 1000, size=(200, D)).astype(np.int64)
    H = scipy.linalg.hadamard(D).astype(np.int64)
    got = oracle_mod.fwht_f32(x.astype(np.float32))
    assert np.array_equal(got.astype(np.int64), x @ H)
    twice = oracle_mod.fwht_f32(got)
    assert np.array_equal(twice.astype(np.int64), D * x)


@pytest.mark.parametrize("D", [64, 128])
def test_fwht_unit_vectors_give_rows(oracle_mod, D):
    got = oracle_mod.fwht_f32(np.eye(D, dtype=np.float32))
    assert np.array_equal(got, scipy.linalg.hadamard(D).astype(np.float32))


@pytest.mark.parametrize("D", [64, 128])
def test_fwht_fp32_error_bound(oracle_mod, D):
    rng = np.random.default_rng(3 + D)
    x = (rng.standard_normal((500, D)) * np.exp(rng.standard_normal((500, 1)) * 3)).astype(np.float32)
    H = scipy.linalg.hadamard(D).astype(np.float64)
    exact = x.astype(np.float64) @ H
    got = oracle_mod.fwht_f32(x).astype(np.float64)
    # each of the log2(D) stages adds at most one rounding of relative size
    # 2^-24 to partial sums bounded by sum|x|
    bound = 1.01 * math.log2(D) * 2.0 ** -24 * np.abs(x.astype(np.float64)).sum(axis=1, keepdims=True)
    assert (np.abs(got - exact) <= bound).all()
