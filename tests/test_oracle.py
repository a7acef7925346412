"""Pins of the fp64 CPU oracle against things other than itself.

* a dense brute force built from the note's mask view (tests/dense_ref.py),
  over a sweep of tiny shapes with windows, dilation, duplicates, padding;
* full attention (torch SDPA, fp64) when the window covers everything;
* global rows equal full attention over the non-padded keys;
* softmax rows sum to one and are supported exactly on K(i);
* K(i) = window U G for dilation 1, built here from Python sets;
* closed-form key totals of the five workloads, derived by hand below;
* values stated by the pages (tests/golden/page_examples.json);
* special inputs: Q = 0 gives the mean of V over K(i); constant V gives the
  constant; one-hot V columns read off the probabilities.
"""
import json
import os

import numpy as np
import pytest
import torch

import oracle
from sparse_long_sequence_fwd_b200 import flops, workloads
from tests.dense_ref import dense_forward, dense_mask

GOLDEN = json.load(open(os.path.join(os.path.dirname(__file__), "golden", "page_examples.json")))


def _rand(shape, seed):
    g = torch.Generator().manual_seed(seed)
    return torch.randn(shape, generator=g)


# ---------------------------------------------------------------- dense pin
def _sweep_cases():
    rng = np.random.default_rng(12345)
    cases = []
    for n in range(60):
        T = int(rng.integers(1, 81))
        r = int(rng.integers(0, T + 3))
        dil = [int(rng.integers(1, 4)) for _ in range(2)]
        B = int(rng.integers(1, 3))
        ng = int(rng.integers(0, 5))
        G = None
        if ng:
            # duplicates, edges and out-of-range entries on purpose
            G = rng.integers(-2, T + 2, size=(B, ng)).astype(np.int32)
            G[:, 0] = T - 1
        pad = None
        if rng.random() < 0.5:
            pad = (rng.random((B, T)) < 0.3).astype(np.uint8)
            if rng.random() < 0.2:
                pad[0, :] = 1  # an all-padded sample
        d = int(rng.choice([1, 3, 8, 16]))
        cases.append((T, r, dil, B, G, pad, d, n))
    return cases


@pytest.mark.parametrize("case", _sweep_cases())
def test_oracle_matches_dense_mask_view(case):
    T, r, dil, B, G, pad, d, seed = case
    H = 2
    q, k, v = (_rand((B, H, T, d), seed * 3 + j) for j in range(3))
    scale = 0.7
    ours = oracle.fwd(q, k, v, r, dil=dil, global_idx=G, key_pad_mask=pad, scale=scale)
    ref = dense_forward(q.double().numpy(), k.double().numpy(), v.double().numpy(), r,
                        dil, G, pad, scale)
    np.testing.assert_allclose(ours, ref, rtol=0, atol=1e-12)


# ------------------------------------------------------- full attention pin
@pytest.mark.parametrize("T,d", [(1, 4), (17, 8), (64, 16), (130, 32)])
def test_window_covering_all_is_full_attention(T, d):
    B, H = 2, 3
    q, k, v = (_rand((B, H, T, d), 100 + j) for j in range(3))
    scale = 1.0 / np.sqrt(d)
    ours = oracle.fwd(q, k, v, r=T, scale=scale)
    sdpa = torch.nn.functional.scaled_dot_product_attention(q.double(), k.double(), v.double(),
                                                            scale=scale)
    np.testing.assert_allclose(ours, sdpa.numpy(), rtol=0, atol=1e-12)


def test_global_rows_are_full_attention_over_unpadded_keys():
    B, H, T, d = 2, 2, 50, 8
    q, k, v = (_rand((B, H, T, d), 200 + j) for j in range(3))
    G = np.array([[3, 49, 20], [0, 0, 11]], dtype=np.int32)
    pad = np.zeros((B, T), dtype=np.uint8)
    pad[1, 40:] = 1
    pad[0, 20] = 1  # a padded global: still a global query, never a key
    ours = oracle.fwd(q, k, v, r=2, dil=[1, 2], global_idx=G, key_pad_mask=pad, scale=0.3)
    for b in range(B):
        keep = torch.from_numpy(pad[b] == 0)
        sd = torch.nn.functional.scaled_dot_product_attention(
            q[b].double(), k[b].double(), v[b].double(), attn_mask=keep[None, None, :].expand(H, T, T),
            scale=0.3)
        for g in set(G[b].tolist()):
            np.testing.assert_allclose(ours[b, :, g], sd[:, g].numpy(), rtol=0, atol=1e-12)


# --------------------------------------------------------- row-sum / support
def test_rows_sum_to_one_on_exact_support():
    B, H, T, d = 2, 2, 45, 4
    q, k, v = (_rand((B, H, T, d), 300 + j) for j in range(3))
    G = np.array([[5, 44], [9, 9]], dtype=np.int32)
    pad = np.zeros((B, T), dtype=np.uint8)
    pad[1, 30:] = 1
    dil = [1, 3]
    for b in range(B):
        for h in range(H):
            for i in range(T):
                probs, _ = oracle.row_probs(q, k, v, 4, b, h, i, dil=dil, global_idx=G,
                                            key_pad_mask=pad, scale=0.5)
                allowed = dense_mask(T, 4, dil[h], G[b].tolist(), pad[b])[i]
                assert np.all((probs > 0) == allowed)
                if allowed.any():
                    assert abs(probs.sum() - 1.0) < 1e-12


def test_key_set_is_window_union_globals_for_dilation_one():
    spec = GOLDEN["global_row"]
    T, r, G = spec["T"], spec["r"], spec["G"]
    for i in range(T):
        ks = set(oracle.key_set(T, r, 1, i, G).tolist())
        if i in G:
            assert ks == set(range(T))
        else:
            window = {j for j in range(i - r, i + r + 1) if 0 <= j < T}
            assert ks == window | set(G)


# ------------------------------------------------------ closed-form totals
def _closed_form_total_no_globals(T, r):
    """Sum_i |window(i)| for dil 1, no globals, T > 2r: T(2r+1) - r(r+1)
    (each of the r first and r last rows loses 1 + 2 + ... + r keys)."""
    return T * (2 * r + 1) - r * (r + 1)


@pytest.mark.parametrize("T,r", [(64, 4), (100, 7), (4096, 256), (300, 100)])
def test_closed_form_window_totals(T, r):
    assert oracle.key_total(T, r, 1) == _closed_form_total_no_globals(T, r)


def test_workload_key_totals_closed_form():
    """Hand derivations of sum |N(i)| per head for the tiny and base workloads.

    base (T=4096, r=256, G={0}): row 0 is global (4096 keys); rows 1..256
    contain key 0 in their window, |N| = i + 257 (sum 98,688); rows
    257..3839 have 513 window keys + key 0 = 514 (3583 rows); rows
    3840..4095 have 4352 - i window keys + key 0 (sum 98,688).  Total
    2,043,134.  Spot rows: 1 -> 258, 256 -> 513, 300 -> 514, 4095 -> 258.

    tiny (T=64, r=4, G={0,37}): window total 64*9 - 20 = 556; rows 0 and 37
    are global (64 each, replacing 5 and 9 window keys); key 0 lies in the
    windows of rows 1..4 only, so 64-2-4 = 58 other rows gain it; key 37 lies
    in the windows of rows 33..41 except 37 itself (8 rows), so 62-8 = 54
    rows gain it; 556 - 5 - 9 + 128 + 58 + 54 = 782.
    """
    assert oracle.key_total(64, 4, 1, [0, 37]) == 782
    assert oracle.key_total(4096, 256, 1, [0]) == 2043134
    for i, n in [(0, 4096), (1, 258), (256, 513), (300, 514), (4095, 258)]:
        assert oracle.key_set(4096, 256, 1, i, [0]).size == n


def test_qa_and_dilated_totals_closed_form():
    """qa, sample 0 (T=4096, r=256, G=0..63, no padding): 64 global rows of
    4096; rows 64..319 have |N| = i + 257 (globals inside or just outside the
    window make up the clipped/overlapping part; sum 114,816); rows
    320..3839 have 513 + 64 = 577 (3520 rows); rows 3840..4095 have
    4416 - i (sum 114,816).  Total 2,522,816.

    qa, sample 1 (keys 3001.. padded): 64 global rows of 3001; rows 64..319
    give i + 257 (114,816); rows 320..2744 give 577 (2425 rows); rows
    2745..3256 keep window keys up to 3000: 3321 - i (164,096); rows
    3257..4095 keep only the 64 globals (839 rows).  Total 1,923,897.

    dilated, dil 1 head (T=8192, r=128, G={0}): 8192 + sum_{1..128}(i+129)
    + 7935*258 + sum_{8064..8191}(8321-i) = 2,104,958.

    dilated, dil 2 head: even class of 4096 (holds key 0): row 0 global
    (8192), the others sum to 4096*257 - 128*129 - 129 window keys plus key 0
    for the 3967 rows beyond its reach; odd class: 4096*257 - 128*129 window
    keys plus key 0 for all 4096 rows.  Total 2,088,446.
    """
    G = list(range(64))
    assert oracle.key_total(4096, 256, 1, G) == 2522816
    pad = np.zeros(4096, dtype=np.uint8)
    pad[3001:] = 1
    assert oracle.key_total(4096, 256, 1, G, pad) == 1923897
    assert oracle.key_total(8192, 128, 1, [0]) == 2104958
    assert oracle.key_total(8192, 128, 2, [0]) == 2088446


def test_qa_padded_sample_totals():
    """qa workload, sample 1: keys 3001..4095 padded, G = 0..63.

    Row 3001 (padded query, not global): window [2745, 3257] keeps 2745..3000
    (256 keys) plus the 64 globals = 320.  Row 4095: window [3839, 4095] is
    all padded, so only the 64 globals remain.
    """
    pad = np.zeros(4096, dtype=np.uint8)
    pad[3001:] = 1
    G = list(range(64))
    assert oracle.key_set(4096, 256, 1, 3001, G, pad).size == 320
    assert oracle.key_set(4096, 256, 1, 4095, G, pad).size == 64
    assert oracle.key_set(4096, 256, 1, 5, G, pad).size == 3001  # global row


def test_flop_counter_matches_oracle_key_sets():
    rng = np.random.default_rng(7)
    for _ in range(25):
        T = int(rng.integers(1, 200))
        r = int(rng.integers(0, 40))
        dil = int(rng.integers(1, 5))
        G = rng.integers(-1, T + 1, size=int(rng.integers(0, 6))).tolist()
        pad = (rng.random(T) < 0.2).astype(np.uint8) if rng.random() < 0.5 else None
        counts = flops.row_key_counts(T, r, dil, G, pad)
        for i in range(T):
            assert counts[i] == oracle.key_set(T, r, dil, i, G, pad).size
        assert counts.sum() == oracle.key_total(T, r, dil, G, pad)


@pytest.mark.parametrize("w", workloads.ALL[:4], ids=lambda w: w.name)
def test_flop_counter_matches_oracle_on_workloads(w):
    inp = workloads.make_inputs(w)
    G = inp["global_idx"]
    pad = inp["key_pad_mask"]
    total = 0
    for b in range(w.B):
        for h in range(w.H):
            total += oracle.key_total(w.T, w.r, int(w.dil[h]),
                                      None if G is None else G[b].numpy(),
                                      None if pad is None else pad[b].numpy())
    assert total == flops.total_keys(w.B, w.H, w.T, w.r, w.dil, G, pad)


# ----------------------------------------------------------- page examples
def test_page_window_size():
    for c in GOLDEN["window_size"]["cases"]:
        T = 4 * c["r"] + 8
        i = T // 2
        assert oracle.key_set(T, c["r"], 1, i).size == c["w"]


def test_page_dilation_reach():
    spec = GOLDEN["dilation_reach"]
    T = 4 * spec["span"]
    i = T // 2
    ks = oracle.key_set(T, spec["r"], spec["dil"], i)
    assert ks.size == spec["keys_per_interior_row"]
    assert ks.max() - ks.min() == spec["span"]


def test_page_dilation_offsets():
    spec = GOLDEN["dilation_offsets"]
    T, i = 200, 100
    offs = set(np.abs(oracle.key_set(T, 10, spec["dil"], i) - i).tolist())
    assert set(spec["first_offsets"]) <= offs
    assert not (set(spec["excluded_offsets"]) & offs)


def test_page_linear_scaling():
    spec = GOLDEN["linear_scaling"]
    a, b = spec["T_from"], spec["T_to"]
    assert (b * b) // (a * a) == spec["dense_factor"]
    r = 8  # fixed window: total = T(2r+1) - r(r+1); the edge rows keep it just above 16
    ratio = oracle.key_total(b, r, 1) / oracle.key_total(a, r, 1)
    assert spec["sparse_factor"] <= ratio < spec["sparse_factor"] + 0.2


# ----------------------------------------------------------- special inputs
def test_zero_queries_give_mean_of_values_over_key_set():
    B, H, T, d = 1, 2, 37, 5
    q = torch.zeros(B, H, T, d)
    k, v = _rand((B, H, T, d), 401), _rand((B, H, T, d), 402)
    G = np.array([[2, 30]], dtype=np.int32)
    pad = np.zeros((B, T), dtype=np.uint8)
    pad[0, 10:13] = 1
    dil = [2, 1]
    out = oracle.fwd(q, k, v, 3, dil=dil, global_idx=G, key_pad_mask=pad, scale=1.0)
    for h in range(H):
        for i in range(T):
            ks = oracle.key_set(T, 3, dil[h], i, G[0], pad[0])
            np.testing.assert_allclose(out[0, h, i], v[0, h, ks].double().mean(0).numpy(),
                                       rtol=0, atol=1e-12)


def test_constant_values_give_the_constant():
    B, H, T, d = 2, 1, 29, 3
    q, k = _rand((B, H, T, d), 501), _rand((B, H, T, d), 502)
    v = torch.full((B, H, T, d), 0.375)
    out = oracle.fwd(q, k, v, 2, dil=[3], global_idx=np.array([[4], [28]], np.int32), scale=2.0)
    np.testing.assert_allclose(out, 0.375, rtol=0, atol=1e-14)


def test_one_hot_values_read_off_probabilities():
    B, H, T = 1, 1, 12
    d = T
    q, k = _rand((B, H, T, 4), 601), _rand((B, H, T, 4), 602)
    # head dim of v may differ from q/k in general; here pass d = T by
    # zero-extending q/k, which leaves the scores unchanged
    qz = torch.zeros(B, H, T, d)
    kz = torch.zeros(B, H, T, d)
    qz[..., :4] = q
    kz[..., :4] = k
    v = torch.eye(T).reshape(1, 1, T, T)
    G = np.array([[7]], np.int32)
    out = oracle.fwd(qz, kz, v, 2, dil=[1], global_idx=G, scale=0.9)
    for i in range(T):
        probs, _ = oracle.row_probs(qz, kz, v, 2, 0, 0, i, dil=[1], global_idx=G, scale=0.9)
        np.testing.assert_allclose(out[0, 0, i], probs, rtol=0, atol=1e-14)


def test_empty_key_set_gives_zero():
    B, H, T, d = 1, 1, 10, 4
    q, k, v = (_rand((B, H, T, d), 700 + j) for j in range(3))
    pad = np.ones((B, T), dtype=np.uint8)
    out = oracle.fwd(q, k, v, 3, key_pad_mask=pad, global_idx=np.array([[2]], np.int32))
    assert np.all(out == 0.0)
