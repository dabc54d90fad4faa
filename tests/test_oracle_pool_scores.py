"""Pins of the oracle's pooling and scoring steps (no GPU): closed forms, special
cases that reduce to a library GEMM, and the parameter count the pages print."""
import os

import numpy as np
import pytest

from oracle import veda_oracle as O

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _golden(name):
    vals = {}
    for line in open(os.path.join(GOLDEN, name)):
        line = line.split("#")[0].strip()
        if line:
            k, v = line.split("=")
            vals[k.strip()] = int(v)
    return vals


def _tiles(n_valid_list, D=128, fill=None, seed=0):
    rng = np.random.default_rng(seed)
    nT = len(n_valid_list)
    x = rng.standard_normal((1, 1, nT * 128, D)) if fill is None else fill.copy()
    return x, np.array([n_valid_list])


def test_pool_constant_tile():
    x = np.full((1, 1, 256, 128), 3.25)
    p = O.pool(x, np.array([[128, 17]]))
    assert (p == 3.25).all()


def test_pool_ramp_closed_form():
    # slot i of the tile holds the value i in every channel: mean (n-1)/2, max n-1, min 0
    for n in (1, 2, 17, 100, 128):
        x = np.zeros((1, 1, 128, 128))
        x[0, 0, :, :] = np.arange(128)[:, None]
        p = O.pool(x, np.array([[n]]))
        assert np.allclose(p[0, 0, 0, 0], (n - 1) / 2, rtol=0, atol=1e-12)
        assert (p[0, 0, 0, 1] == n - 1).all() and (p[0, 0, 0, 2] == 0).all()


def test_pool_ignores_pads_and_is_order_invariant():
    x, nv = _tiles([40, 128])
    p = O.pool(x, nv)
    y = x.copy()
    y[0, 0, 40:128] = 1e6                       # garbage in the pad slots of tile 0
    perm = np.random.default_rng(3).permutation(40)
    y[0, 0, :40] = x[0, 0, perm]                # shuffle the valid slots
    assert np.allclose(O.pool(y, nv), p, rtol=1e-14, atol=1e-14)


def test_pool_empty_tile_is_zero():
    x, _ = _tiles([1, 1])
    p = O.pool(x, np.array([[5, 0]]))
    assert (p[0, 0, 1] == 0).all()


def _pooled(seed, B=2, H=3, nT=5):
    rng = np.random.default_rng(seed)
    return rng.standard_normal((B, H, nT, 3, 128))


def test_scores_zero_weights_is_gemm_of_means():
    pq, pk = _pooled(0), _pooled(1)
    W0 = np.zeros((3, 128, 384))
    S = O.scores(pq, pk, W0, W0)
    for b in range(2):
        for h in range(3):
            ref = np.matmul(pq[b, h, :, 0, :], pk[b, h, :, 0, :].T)
            assert np.allclose(S[b, h], ref, rtol=1e-13, atol=1e-12)


def test_scores_selector_weights_closed_forms():
    pq, pk = _pooled(2), _pooled(3)
    I, Z = np.eye(128), np.zeros((128, 128))
    W_mean = np.tile(np.concatenate([I, Z, Z], axis=1), (3, 1, 1))     # qhat = 2 mean
    W_max = np.tile(np.concatenate([Z, I, Z], axis=1), (3, 1, 1))      # khat = mean + max
    S = O.scores(pq, pk, W_mean, W_max)
    qh = 2 * pq[:, :, :, 0]
    kh = pk[:, :, :, 0] + pk[:, :, :, 1]
    assert np.allclose(S, np.matmul(qh, np.swapaxes(kh, -1, -2)), rtol=1e-13, atol=1e-11)
    W_min = np.tile(np.concatenate([Z, Z, -I], axis=1), (3, 1, 1))     # qhat = mean - min
    S2 = O.scores(pq, pk, W_min, np.zeros((3, 128, 384)))
    qh2 = pq[:, :, :, 0] - pq[:, :, :, 2]
    assert np.allclose(S2, np.matmul(qh2, np.swapaxes(pk[:, :, :, 0], -1, -2)), rtol=1e-13, atol=1e-11)


def test_scores_affine_in_weights_and_per_head():
    rng = np.random.default_rng(5)
    pq, pk = _pooled(6), _pooled(7)
    Wk = 0.02 * rng.standard_normal((3, 128, 384))
    A, Bm = 0.02 * rng.standard_normal((2, 3, 128, 384))
    Z = np.zeros_like(A)
    lhs = O.scores(pq, pk, A + Bm, Wk) + O.scores(pq, pk, Z, Wk)
    rhs = O.scores(pq, pk, A, Wk) + O.scores(pq, pk, Bm, Wk)
    assert np.allclose(lhs, rhs, rtol=1e-11, atol=1e-10)
    # head h only uses W[h]
    A2 = A.copy()
    A2[1] += 1.0
    d = O.scores(pq, pk, A2, Wk) - O.scores(pq, pk, A, Wk)
    assert np.abs(d[:, [0, 2]]).max() == 0 and np.abs(d[:, 1]).max() > 0


def test_predictor_parameter_count_matches_the_pages():
    g = _golden("predictor_size.txt")
    n = O.predictor_param_count(g["attention_heads"], g["transformer_blocks"], g["head_dim"])
    assert n == 275_251_200
    assert round(n / 1e6) == g["params_total_millions"]
    # one byte per parameter in the fp8 bundle is 262.5 MiB; the bundle also carries its
    # small plan tables, and is printed as 263 MB
    assert n / 2 ** 20 <= g["bundle_megabytes"] < n / 2 ** 20 + 1
    # a bias per projection output would push it to 276M, so the reading is bias-free
    assert round((n + 2 * 128 * g["attention_heads"] * g["transformer_blocks"]) / 1e6) != 275
