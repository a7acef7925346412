"""Pins of the oracle's backward (oracle.bwd) against things other than
itself: central finite differences of the C oracle's forward, and closed
forms (sum_j dv_j = sum_i dy_i over rows that have keys; sum_j dk_j = 0 per
(b, h), since every row's ds sums to zero; dy = 0 gives zero gradients)."""
import numpy as np
import pytest
import torch

import oracle


def _case(seed, B=1, H=2, T=23, d=4):
    g = torch.Generator().manual_seed(seed)
    return [torch.randn(B, H, T, d, generator=g, dtype=torch.float64).float() for _ in range(4)]


@pytest.mark.parametrize("seed,r,dil,G,pad_from", [(1, 3, [1, 2], [[0, 11, 11]], None),
                                                   (2, 2, [2, 1], [[22, 5]], 18),
                                                   (3, 30, [1, 1], None, None)])
def test_backward_matches_finite_differences(seed, r, dil, G, pad_from):
    q, k, v, dy = _case(seed)
    T = q.shape[2]
    Gt = None if G is None else np.asarray(G, dtype=np.int32)
    pad = None
    if pad_from is not None:
        pad = np.zeros((1, T), dtype=np.uint8)
        pad[0, pad_from:] = 1
    dq, dk, dv = oracle.bwd(q, k, v, dy, r, dil=dil, global_idx=Gt, key_pad_mask=pad, scale=0.7)
    f = lambda qq, kk, vv: float((oracle.fwd(qq, kk, vv, r, dil=dil, global_idx=Gt, key_pad_mask=pad,
                                             scale=0.7) * dy.double().numpy()).sum())
    rng = np.random.default_rng(seed)
    eps = 1e-3
    for which, grad in ((0, dq), (1, dk), (2, dv)):
        U = rng.standard_normal(q.shape).astype(np.float32)
        args_p = [x.double().numpy().astype(np.float32) for x in (q, k, v)]
        args_m = [a.copy() for a in args_p]
        # fp32 inputs of the C oracle: perturb in fp64, store the exact fp32 steps taken
        xp = args_p[which].astype(np.float64) + eps * U
        xm = args_p[which].astype(np.float64) - eps * U
        args_p[which] = xp.astype(np.float32)
        args_m[which] = xm.astype(np.float32)
        step = args_p[which].astype(np.float64) - args_m[which].astype(np.float64)
        fd = (f(*args_p) - f(*args_m))
        pred = float((grad * step).sum())
        assert fd == pytest.approx(pred, rel=1e-5, abs=1e-9)


def test_backward_closed_forms():
    q, k, v, dy = _case(7, B=2, H=2, T=40, d=6)
    G = np.array([[3, 39], [0, 0]], dtype=np.int32)
    pad = np.zeros((2, 40), dtype=np.uint8)
    pad[1, 30:] = 1
    dq, dk, dv = oracle.bwd(q, k, v, dy, 4, dil=[1, 3], global_idx=G, key_pad_mask=pad, scale=0.5)
    # every row here has keys, so sum_j dv_j = sum_i dy_i and sum_j dk_j = 0
    np.testing.assert_allclose(dv.sum(axis=2), dy.double().numpy().sum(axis=2), rtol=0, atol=1e-12)
    np.testing.assert_allclose(dk.sum(axis=2), 0.0, rtol=0, atol=1e-12)
    # padded keys get no gradient
    assert np.all(dk[1, :, 30:] == 0) and np.all(dv[1, :, 30:] == 0)
    z = oracle.bwd(q, k, v, torch.zeros_like(dy), 4, dil=[1, 3], global_idx=G, key_pad_mask=pad, scale=0.5)
    assert all(np.all(x == 0) for x in z)
