"""Pins of the oracle's random-block rule (the BigBird variant) against
things other than itself.

Rule (mhpn.cn page, sections 2.2.1 and 2.2.2; aiqz.cc page, BigBird
comparison): an ordinary row i also keeps the keys of the n_rand key blocks
of 64 drawn for its query block i // 64; blocks outside the sequence are
ignored; the key set stays a set.  Global rows are unchanged.

* a dense brute force: the mask view's membership rule plus the random
  blocks, built here with numpy broadcasting, over a sweep of tiny shapes;
* every key block drawn for every query block: full attention over the
  non-padded keys (torch SDPA, fp64);
* no draws, or only out-of-range draws: the plain oracle, bit for bit;
* a hand-counted case: with Q = 0 the weights are uniform over K(i), so a
  V column holding the key index reads off the mean key index of K(i).
"""
import numpy as np
import pytest
import torch

import oracle
from tests.dense_ref import dense_attention, dense_mask

BLK = 64


def _rand(shape, seed):
    g = torch.Generator().manual_seed(seed)
    return torch.randn(shape, generator=g)


def _dense_rand_forward(q, k, v, r, dil, G, pad, scale, rb):
    """q, k, v fp64 numpy [B, H, T, d]; rb int [B, H, nqb, n_rand]."""
    B, H, T, d = q.shape
    out = np.zeros_like(q)
    i = np.arange(T)
    for b in range(B):
        Gb = [] if G is None else list(np.asarray(G)[b])
        padb = None if pad is None else np.asarray(pad)[b]
        g = np.zeros(T, dtype=bool)
        for x in Gb:
            if 0 <= x < T:
                g[x] = True
        for h in range(H):
            allowed = dense_mask(T, r, int(dil[h]), Gb, None)
            # key block of column j is one of the draws of row i's query block
            draws = np.asarray(rb[b, h])[i // BLK]                      # [T, n_rand]
            hit = (draws[:, :, None] == (i // BLK)[None, None, :]).any(axis=1)  # [T, T]
            allowed = allowed | (hit & ~g[:, None])                     # global rows already keep every key
            if padb is not None:
                allowed &= ~np.asarray(padb, dtype=bool)[None, :]
            out[b, h] = dense_attention(q[b, h], k[b, h], v[b, h], allowed, scale)
    return out


def _sweep():
    rng = np.random.default_rng(777)
    cases = []
    for n in range(30):
        T = int(rng.integers(1, 300))
        nqb = (T + BLK - 1) // BLK
        r = int(rng.integers(0, 40))
        dil = [int(rng.integers(1, 3)) for _ in range(2)]
        B = int(rng.integers(1, 3))
        n_rand = int(rng.integers(1, 4))
        # in-range draws, duplicates and out-of-range entries on purpose
        rb = rng.integers(-1, nqb + 1, size=(B, 2, nqb, n_rand)).astype(np.int32)
        G = None
        if rng.random() < 0.6:
            G = rng.integers(0, T, size=(B, int(rng.integers(1, 4)))).astype(np.int32)
        pad = None
        if rng.random() < 0.5:
            pad = (rng.random((B, T)) < 0.2).astype(np.uint8)
        d = int(rng.choice([2, 8]))
        cases.append((T, r, dil, B, G, pad, d, rb, n))
    return cases


@pytest.mark.parametrize("case", _sweep())
def test_random_blocks_match_dense_brute_force(case):
    T, r, dil, B, G, pad, d, rb, seed = case
    H = 2
    q, k, v = (_rand((B, H, T, d), 5000 + seed * 3 + j) for j in range(3))
    ours = oracle.fwd(q, k, v, r, dil=dil, global_idx=G, key_pad_mask=pad, scale=0.6, rand_blocks=rb)
    ref = _dense_rand_forward(q.double().numpy(), k.double().numpy(), v.double().numpy(), r, dil, G, pad, 0.6, rb)
    np.testing.assert_allclose(ours, ref, rtol=0, atol=1e-12)


@pytest.mark.parametrize("T", [64, 200])
def test_all_blocks_drawn_is_full_attention(T):
    B, H, d = 2, 2, 8
    q, k, v = (_rand((B, H, T, d), 6000 + j) for j in range(3))
    nqb = (T + BLK - 1) // BLK
    rb = np.broadcast_to(np.arange(nqb, dtype=np.int32), (B, H, nqb, nqb)).copy()
    pad = np.zeros((B, T), dtype=np.uint8)
    pad[1, T // 2:] = 1
    ours = oracle.fwd(q, k, v, 1, key_pad_mask=pad, scale=0.5, rand_blocks=rb)
    for b in range(B):
        keep = torch.from_numpy(pad[b] == 0)
        sd = torch.nn.functional.scaled_dot_product_attention(
            q[b].double(), k[b].double(), v[b].double(), attn_mask=keep[None, None, :].expand(H, T, T), scale=0.5)
        np.testing.assert_allclose(ours[b], sd.numpy(), rtol=0, atol=1e-12)


def test_no_or_out_of_range_draws_give_the_plain_oracle():
    B, H, T, d = 1, 2, 150, 8
    q, k, v = (_rand((B, H, T, d), 7000 + j) for j in range(3))
    G = np.array([[7, 140]], dtype=np.int32)
    plain = oracle.fwd(q, k, v, 10, dil=[1, 2], global_idx=G, scale=0.4)
    nqb = (T + BLK - 1) // BLK
    bad = np.full((B, H, nqb, 2), -1, dtype=np.int32)
    bad[..., 1] = nqb  # past the last block
    assert np.array_equal(oracle.fwd(q, k, v, 10, dil=[1, 2], global_idx=G, scale=0.4, rand_blocks=bad), plain)


def test_hand_counted_key_sets():
    """Q = 0: uniform weights over K(i); V[:, 0] = 1, V[:, 1] = j, so y_i =
    (1, mean of K(i)).  T = 130 (query blocks 0, 1 and a two-row block 2),
    r = 0, no globals: K(i) = {i} U the drawn blocks."""
    T = 130
    q = torch.zeros(1, 1, T, 2)
    k = _rand((1, 1, T, 2), 8000)
    v = torch.zeros(1, 1, T, 2)
    v[0, 0, :, 0] = 1.0
    v[0, 0, :, 1] = torch.arange(T, dtype=torch.float32)
    rb = np.array([[[[1, 1], [-1, 5], [0, 2]]]], dtype=np.int32)  # [1, 1, 3 query blocks, 2]
    y = oracle.fwd(q, k, v, 0, scale=1.0, rand_blocks=rb)[0, 0]
    # row 5 (block 0 draws block 1 twice): {5} U [64, 128): 65 keys
    assert y[5, 0] == pytest.approx(1.0)
    assert y[5, 1] == pytest.approx((5 + sum(range(64, 128))) / 65, abs=1e-12)
    # row 100 (block 1 draws nothing in range): {100}
    assert y[100, 1] == pytest.approx(100.0, abs=1e-12)
    # row 70 lies inside its own drawn block?  block 1 drew nothing: {70}
    assert y[70, 1] == pytest.approx(70.0, abs=1e-12)
    # row 129 (block 2 draws blocks 0 and 2): [0, 64) U {128, 129}: 66 keys
    assert y[129, 1] == pytest.approx((sum(range(64)) + 128 + 129) / 66, abs=1e-12)
    # row 60 (block 0, drawn block 1 is [64, 128)): its own row 60 is in the window
    assert y[60, 1] == pytest.approx((60 + sum(range(64, 128))) / 65, abs=1e-12)


def test_flop_counter_counts_random_keys():
    """The benchmark's key counter (flops.row_key_counts + rand_extra_counts)
    against the brute-force membership rule above."""
    from sparse_long_sequence_fwd_b200 import flops
    rng = np.random.default_rng(3)
    for _ in range(20):
        T = int(rng.integers(1, 300))
        r = int(rng.integers(0, 40))
        nqb = (T + BLK - 1) // BLK
        rb = rng.integers(-1, nqb + 1, size=(nqb, 3))
        G = rng.integers(0, T, size=2) if rng.random() < 0.5 else None
        pad = (rng.random(T) < 0.2) if rng.random() < 0.5 else None
        got = flops.row_key_counts(T, r, 1, G, pad) + flops.rand_extra_counts(T, r, G, pad, rb)
        i = np.arange(T)
        g = np.zeros(T, dtype=bool)
        if G is not None:
            g[G] = True
        allowed = (np.abs(i[:, None] - i[None, :]) <= r) | g[None, :] | g[:, None]
        allowed |= (rb[i // BLK][:, :, None] == (i // BLK)[None, None, :]).any(axis=1)
        if pad is not None:
            allowed &= ~pad[None, :]
        assert np.array_equal(got, allowed.sum(axis=1))
