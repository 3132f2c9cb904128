"""Pins for the oracle's codebook linear layer.

Source: rcap.io summary, rotation-cancellation paragraph (W R^T R x = W x) and the
pseudocode's W_hat = diag(row_norms) nearest_centroid(.), x_hat = s nearest_centroid(.):
y[t,o] = s_t rn_o sum_k sigma ca[xc] sigma cw[wc].  Pinned against a dense numpy matrix
product of codes decoded with numpy's own bit unpacking, a closed form for constant codes,
and the quantized layer approaching W x as bits grow.
"""
import numpy as np
import pytest

import oracle as O
from calibration_free_bit_b200 import synth
from test_oracle_quantize import unpack_numpy


@pytest.mark.parametrize("ba,bw", [(4, 4), (4, 2), (4, 3), (8, 4)])
def test_linear_matches_dense_matmul(ba, bw):
    rng = np.random.default_rng(ba * 10 + bw)
    T, d, out = 9, 256, 23
    xc = rng.integers(0, 1 << ba, (T, d)).astype(np.uint8)
    wc = rng.integers(0, 1 << bw, (out, d)).astype(np.uint8)
    s = rng.uniform(0.5, 3.0, T)
    rn = rng.uniform(0.1, 2.0, out)
    xp, wp = O.pack(xc, ba), O.pack(wc, bw)
    ca, _ = O.codebook(ba)
    cw, _ = O.codebook(bw)
    sig = 1.0 / np.sqrt(d)
    A = sig * ca[unpack_numpy(xp, d, ba)]
    B = sig * cw[unpack_numpy(wp, d, bw)]
    want = s[:, None] * rn[None, :] * (A @ B.T)
    np.testing.assert_allclose(O.linear(xp, s, wp, rn, d, ba, bw), want, rtol=1e-12,
                               atol=1e-14)


def test_linear_constant_codes_closed_form():
    """All activation codes i, all weight codes j: y = s rn d sigma^2 ca[i] cw[j]
    = s rn ca[i] cw[j]."""
    d = 128
    ca, _ = O.codebook(4)
    cw, _ = O.codebook(2)
    for i, j in [(0, 3), (7, 1), (15, 0), (8, 2)]:
        xp = O.pack(np.full((1, d), i, np.uint8), 4)
        wp = O.pack(np.full((1, d), j, np.uint8), 2)
        y = O.linear(xp, [2.5], wp, [0.75], d, 4, 2)[0, 0]
        assert y == pytest.approx(2.5 * 0.75 * ca[i] * cw[j], rel=1e-13)


def test_quantized_linear_approaches_Wx():
    """Sanity (not a bound): relative error of the quantized layer against W x shrinks
    as bits grow."""
    p = synth.get("toy_w4a4")[0]
    x = synth.activations(p).double().numpy()[:32]
    W = synth.weight(p).double().numpy()
    perm, sign = O.build_rpbh(p.d, 0)
    exact = x @ W.T
    errs = []
    for ba, bw in [(4, 2), (4, 4), (8, 8)]:
        xp, s = O.quantize_act(x, p.h, perm, sign, ba)
        wp, rn = O.quantize_weight(W, p.h, perm, sign, bw)
        y = O.linear(xp, s, wp, rn, p.d, ba, bw)
        errs.append(np.linalg.norm(y - exact) / np.linalg.norm(exact))
    assert errs[0] > errs[1] > errs[2]
    assert errs[2] < 0.05
