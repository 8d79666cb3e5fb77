"""Pins of oracle.projection (CPU).

The oracle's projections are matrix products plus reshapes; each is checked here
against a computation that shares neither: scalar loops over every output
element on tiny shapes, written from the definitions in the oracle's header
(q[b,h,l,j] = sum_c x[b,l,c] W[64h+j, c] + bias[64h+j], k and v with the row
offsets C and 2C; y[b,l,n] = sum_{h,j} O[b,h,l,j] W[n, 64h+j] + bias[n]).  A
transposed weight, a swapped q/k/v order, a wrong head offset or a dropped bias
fails one of them.  The magnitudes used for GPU tolerances are pinned the same
way (inflating them would loosen every tolerance unnoticed).
"""

import numpy as np

from oracle import projection as OP


def _rand(rng, *shape):
    return rng.standard_normal(shape)


def test_qkv_projection_against_scalar_loops():
    rng = np.random.default_rng(11)
    B, L, H = 2, 3, 2
    C = 64 * H
    x, w, b = _rand(rng, B, L, C), _rand(rng, 3 * C, C), _rand(rng, 3 * C)
    q, k, v = OP.qkv_projection(x, w, b, H)
    mq, mk, mv = OP.magnitude_qkv(x, w, b, H)
    for which, (got, mag) in enumerate(((q, mq), (k, mk), (v, mv))):
        assert got.shape == (B, H, L, 64)
        for bb in range(B):
            for h in range(H):
                for l in range(L):
                    for j in range(0, 64, 7):
                        row = which * C + 64 * h + j
                        s = b[row]
                        a = abs(b[row])
                        for c in range(C):
                            s += x[bb, l, c] * w[row, c]
                            a += abs(x[bb, l, c] * w[row, c])
                        assert abs(got[bb, h, l, j] - s) < 1e-12 * a
                        assert abs(mag[bb, h, l, j] - a) < 1e-12 * a


def test_out_projection_against_scalar_loops():
    rng = np.random.default_rng(12)
    B, H, L, N = 2, 3, 2, 128
    o, w, b = _rand(rng, B, H, L, 64), _rand(rng, N, 64 * H), _rand(rng, N)
    y = OP.out_projection(o, w, b)
    m = OP.magnitude_out(o, w, b)
    assert y.shape == (B, L, N)
    for bb in range(B):
        for l in range(L):
            for n in range(0, N, 5):
                s = b[n]
                a = abs(b[n])
                for h in range(H):
                    for j in range(64):
                        s += o[bb, h, l, j] * w[n, 64 * h + j]
                        a += abs(o[bb, h, l, j] * w[n, 64 * h + j])
                assert abs(y[bb, l, n] - s) < 1e-12 * a
                assert abs(m[bb, l, n] - a) < 1e-12 * a


def test_split_and_merge_are_inverse_and_no_bias_is_zero_bias():
    rng = np.random.default_rng(13)
    B, L, H = 2, 5, 3
    y = _rand(rng, B, L, 3 * 64 * H)
    q, k, v = OP.split_heads(y, H)
    for i, t in enumerate((q, k, v)):
        assert np.array_equal(OP.merge_heads(t), y[:, :, i * 64 * H:(i + 1) * 64 * H])
    x, w = _rand(rng, B, L, 64 * H), _rand(rng, 64 * H, 64 * H)
    assert np.array_equal(OP.linear(x, w), OP.linear(x, w, np.zeros(64 * H)))
