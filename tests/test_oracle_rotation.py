"""Pins for oracle.rotation: published SplitMix64 outputs, Gaussian moments,
orthogonality, the QR sign convention and rotation invariance of q.k."""
import json
import os

import numpy as np
import pytest

from oracle import rotation

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def test_splitmix64_published_outputs():
    g = json.load(open(os.path.join(GOLDEN, "splitmix64_state0.json")))
    w = rotation.splitmix64_words(g["key"], len(g["outputs_hex"]))
    assert [format(int(x), "016x") for x in w] == g["outputs_hex"]


def test_stream_key_separates_tags_and_sizes():
    assert rotation.stream_key(0, rotation.TAG_KEY, 8) != rotation.stream_key(0, rotation.TAG_VALUE, 8)
    assert rotation.stream_key(0, rotation.TAG_KEY, 8) != rotation.stream_key(0, rotation.TAG_KEY, 10)
    assert rotation.stream_key(5, rotation.TAG_KEY, 8) != rotation.stream_key(0, rotation.TAG_KEY, 8)


def test_gaussian_moments():
    g = rotation.gaussian_matrix(128, rotation.TAG_KEY, 0).ravel()
    assert abs(np.mean(g)) < 0.03
    assert abs(np.var(g) - 1) < 0.04
    assert abs(np.mean(g ** 4) - 3) < 0.2          # Gaussian kurtosis
    assert np.all(np.isfinite(g))


@pytest.mark.parametrize("m", [2, 4, 6, 10, 32, 64, 100, 128])
def test_orthogonal_and_sign_convention(m):
    r = rotation.key_rotation(m, 0)
    assert np.max(np.abs(r @ r.T - np.eye(m))) < 1e-13
    g = rotation.gaussian_matrix(m, rotation.TAG_KEY, 0)
    rr = r.T @ g                                   # the R factor of G = Q R
    assert np.max(np.abs(np.tril(rr, -1))) < 1e-10 * max(1.0, np.max(np.abs(rr)))
    assert np.all(np.diag(rr) > 0)


def test_value_rotation_distinct():
    a = rotation.value_rotation(128, 0)
    b = rotation.key_rotation(128, 0)
    assert np.max(np.abs(a - b)) > 0.1
    assert np.max(np.abs(a @ a.T - np.eye(128))) < 1e-13


def test_rotation_invariance_of_dot():
    rng = np.random.default_rng(0)
    for m in (2, 16, 128):
        r = rotation.key_rotation(m, 3)
        q, k = rng.standard_normal(m), rng.standard_normal(m)
        assert (r @ q) @ (r @ k) == pytest.approx(q @ k, abs=1e-12)


def test_seed_changes_matrix():
    assert np.max(np.abs(rotation.key_rotation(16, 0) - rotation.key_rotation(16, 1))) > 0.1
