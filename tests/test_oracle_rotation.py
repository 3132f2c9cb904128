"""Pins for the oracle's RPBH rotation R = blockdiag(H_h/sqrt h) D P.

Source: rcap.io summary "OrbitQuant: Data-Agnostic Quantization for Image and Video",
RPBH paragraph (permutation, sign flips, block Walsh-Hadamard) and rotation-cancellation
paragraph (R orthogonal, W R^T R x = W x).  Checks use a dense matrix built independently
with numpy (Sylvester recursion by np.kron, a permutation matrix, a diagonal) and the
invariants of an orthogonal map.
"""
import numpy as np
import pytest

import oracle as O
from conftest import golden_rows


def sylvester(h):
    H = np.array([[1]], dtype=np.int64)
    while H.shape[0] < h:
        H = np.block([[H, H], [H, -H]])
    return H


def dense_rotation(d, h, perm, sign):
    P = np.zeros((d, d))
    P[np.arange(d), perm] = 1.0           # (P x)[i] = x[perm[i]]
    D = np.diag(sign.astype(np.float64))
    B = np.kron(np.eye(d // h), sylvester(h) / np.sqrt(h))
    return B @ D @ P


def test_hadamard_order4_golden():
    want = np.array([[int(v) for v in r[0].split()] for r in
                     golden_rows("hadamard_sylvester_h4.txt")])
    assert np.array_equal(O.hadamard(4), want)


@pytest.mark.parametrize("h", [2, 8, 64, 256])
def test_hadamard_matches_sylvester_recursion(h):
    assert np.array_equal(O.hadamard(h), sylvester(h))


@pytest.mark.parametrize("h", [16, 128, 1024])
def test_hadamard_rows_orthogonal(h):
    H = O.hadamard(h) if h <= 128 else sylvester(h)
    if h <= 128:
        assert np.array_equal(H @ H.T, h * np.eye(h, dtype=np.int64))
    # the oracle's entry function on sampled rows of the large order
    if h == 1024:
        rng = np.random.default_rng(0)
        for i in rng.integers(0, h, 6):
            row = np.array([O.lib().orc_hadamard_entry(int(i), j) for j in range(h)])
            assert np.array_equal(row, H[i])


@pytest.mark.parametrize("d,h", [(256, 64), (512, 128), (768, 256), (64, 2)])
def test_rotation_matches_dense_matrix(d, h):
    perm, sign = O.build_rpbh(d, 11)
    R = dense_rotation(d, h, perm, sign)
    x = np.random.default_rng(1).standard_normal((5, d)) * 3.0
    np.testing.assert_allclose(O.rotate(x, h, perm, sign), x @ R.T, rtol=0, atol=1e-12)


def test_rotation_is_orthogonal():
    d, h = 256, 64
    perm, sign = O.build_rpbh(d, 3)
    cols = O.rotate(np.eye(d), h, perm, sign).T      # column k = R e_k
    np.testing.assert_allclose(cols @ cols.T, np.eye(d), atol=1e-14)


def test_rotation_preserves_norm_with_outliers():
    d, h = 3072, 128
    perm, sign = O.build_rpbh(d, 0)
    rng = np.random.default_rng(2)
    x = rng.standard_normal((4, d))
    x[:, rng.choice(d, 31, replace=False)] *= 50.0
    z = O.rotate(x, h, perm, sign)
    np.testing.assert_allclose(np.linalg.norm(z, axis=1), np.linalg.norm(x, axis=1),
                               rtol=1e-14)


def test_spike_spreads_over_exactly_one_block():
    """x = e_k lands on the block holding position perm^-1(k), with |z| = 1/sqrt(h)."""
    d, h = 512, 64
    perm, sign = O.build_rpbh(d, 5)
    inv = np.argsort(perm)
    for k in (0, 17, 511):
        z = O.rotate(np.eye(d)[k], h, perm, sign)[0]
        blk = inv[k] // h
        inside = z[blk * h:(blk + 1) * h]
        np.testing.assert_allclose(np.abs(inside), 1.0 / np.sqrt(h), rtol=1e-15)
        outside = np.delete(z, np.s_[blk * h:(blk + 1) * h])
        assert np.all(outside == 0.0)


def test_weight_rotation_cancels():
    """W R^T R x = W x to 1e-12 (rotation-cancellation paragraph)."""
    d, h, out = 512, 128, 40
    perm, sign = O.build_rpbh(d, 9)
    rng = np.random.default_rng(4)
    W = rng.standard_normal((out, d)) / np.sqrt(d)
    x = rng.standard_normal(d)
    W_rot = O.rotate(W, h, perm, sign)                # rows R w_o, i.e. W R^T
    x_rot = O.rotate(x, h, perm, sign)[0]
    np.testing.assert_allclose(W_rot @ x_rot, W @ x, rtol=0, atol=1e-12)


def test_block_rht_tables_are_rpbh_without_the_permutation():
    """Block-RHT (the ablation): identity permutation, the RPBH signs of the same seed."""
    for d, seed in [(256, 0), (3072, 7)]:
        perm, sign = O.build_rpbh(d, seed)
        pid, sid = O.build_block_rht(d, seed)
        assert np.array_equal(pid, np.arange(d))
        assert np.array_equal(sid, sign)


def test_block_rht_is_orthogonal_and_block_local():
    """With P = I the rotation is blockdiag(H_h/sqrt h) D: orthogonal, and a vector supported
    on one block of positions stays on that block."""
    d, h = 256, 64
    perm, sign = O.build_block_rht(d, 3)
    R = np.stack([O.rotate(e, h, perm, sign)[0] for e in np.eye(d)], axis=1)
    np.testing.assert_allclose(R @ R.T, np.eye(d), atol=1e-13)
    x = np.zeros(d)
    x[h:2 * h] = np.arange(1, h + 1)
    z = O.rotate(x, h, perm, sign)[0]
    assert np.all(z[:h] == 0) and np.all(z[2 * h:] == 0)
    np.testing.assert_allclose(np.linalg.norm(z), np.linalg.norm(x), rtol=1e-14)
