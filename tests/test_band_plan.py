"""The band kernel's work split, checked on the host (no GPU).

The bf16 band kernel walks one sequence of key blocks (per sample, heads;
per head, the residue classes of its dilation; per class, 128-query tiles;
per tile, its band blocks then its global-key blocks, 64 keys each) and
gives every CTA an equal contiguous share of it.  lf_attn_band_plan runs, on the
host, the same walk each pipeline's producer runs on the device.  These
tests check the walk against an independent count of every tile's blocks
(from the window definition: decimated keys [q0 - r, q0 + 127 + r] clipped
to the class, in 64-key blocks counted from q0 - r), and check that the
pieces cover every (tile, block) exactly once, that a split tile's pieces
sit in consecutive pipelines, and that the shares differ by one block at
most.
"""
import numpy as np
import pytest

from sparse_long_sequence_fwd_b200 import build, lf_attn


MAX_CTAS = 296  # the library's cap on band-kernel CTAs (two per SM of a 148-SM B200)


@pytest.fixture(scope="module", autouse=True)
def _lib():
    build.build()
    lf_attn.load()


def expected_tiles(B, H, T, r, dil, n_global):
    """[(bh, c, t, blocks)] in sequence order, from the window definition."""
    r = min(r, T)
    ngb = 0 if n_global == 0 else (min(n_global, T) + 63) // 64
    out = []
    for b in range(B):
        for h in range(H):
            dl = dil[h]
            for c in range(dl):
                Tc = len(range(c, T, dl))
                for t in range((Tc + 127) // 128):
                    q0 = 128 * t
                    lo, hi = max(0, q0 - r), min(Tc - 1, q0 + 127 + r)
                    first = (lo - (q0 - r)) // 64
                    last = (hi - (q0 - r)) // 64
                    out.append((b * H + h, c, t, last - first + 1 + ngb))
    return out


CASES = [
    # B, H, T, r, dil, n_global, pipelines
    (1, 12, 4096, 256, [1] * 12, 1, 296),
    (2, 12, 4096, 256, [1] * 12, 64, 296),
    (1, 12, 8192, 128, [1, 1] + [2] * 10, 1, 296),
    (1, 16, 16384, 256, [1] * 16, 32, 296),
    (1, 2, 64, 4, [1, 1], 2, 296),
    (2, 3, 1000, 100, [1, 2, 3], 4, 296),
    (1, 4, 700, 20, [5, 6, 7, 8], 3, 7),
    (1, 3, 5, 2, [8, 3, 1], 0, 296),          # T < dil: residue classes with no rows
    (1, 2, 400, 100000, [1, 3], 0, 13),       # r far beyond T
    (1, 1, 1, 3, [1], 0, 296),
    (3, 2, 300, 0, [1, 2], 200, 5),           # r = 0, two global blocks per tile
    (1, 12, 4096, 256, [1] * 12, 1, 1),
    (1, 12, 4096, 256, [1] * 12, 1, 301),      # more than the cap
]


@pytest.mark.parametrize("case", CASES, ids=lambda c: "B%d_H%d_T%d_r%d_g%d_p%d" % (c[0], c[1], c[2], c[3], c[5], c[6]))
def test_pieces_cover_every_block_once(case):
    B, H, T, r, dil, ng, pipes = case
    tiles = expected_tiles(B, H, T, r, dil, ng)
    plan = lf_attn.band_plan(B, H, T, r, dil=dil, n_global=ng, max_ctas=pipes)
    n_blocks = sum(t[3] for t in tiles)
    G = min(pipes, MAX_CTAS, n_blocks)
    cover = {}
    for cta, tile, lo, hi, nb, s0, s1, slot, bh, ct in plan.tolist():
        assert 0 <= tile < len(tiles)
        ebh, ec, et, enb = tiles[tile]
        assert (bh, ct >> 16, ct & 0xFFFF, nb) == (ebh, ec, et, enb)
        assert 0 <= lo < hi <= nb
        assert s0 <= cta <= s1 < G
        cover.setdefault(tile, []).append((lo, hi, cta, s0, s1, slot))
    assert sorted(cover) == list(range(len(tiles)))
    slots = []
    for tile, parts in cover.items():
        parts.sort()
        assert parts[0][0] == 0 and parts[-1][1] == tiles[tile][3]
        for a, b in zip(parts, parts[1:]):
            assert a[1] == b[0]          # contiguous, no overlap
            assert b[2] == a[2] + 1      # consecutive pipelines
        s0, s1 = parts[0][3], parts[0][4]
        assert [p[2] for p in parts] == list(range(s0, s1 + 1))
        if len(parts) > 1:
            slots += [p[5] for p in parts]
    assert len(slots) == len(set(slots))
    assert all(0 <= s < 2 * G for s in slots)
    per = np.zeros(G, dtype=np.int64)
    for cta, tile, lo, hi, *_ in plan.tolist():
        per[cta] += hi - lo
    assert per.sum() == n_blocks
    assert per.max() - per.min() <= 1


def test_rejects_bad_sizes():
    with pytest.raises(ValueError):
        lf_attn.band_plan(1, 2, 64, -1)
    with pytest.raises(ValueError):
        lf_attn.band_plan(1, 2, 64, 4, dil=[1, 9])
