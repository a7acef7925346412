"""Helpers shared by the GPU parity tests: run the CUDA path through the
C-ABI binding and the oracle on the same seeded inputs, and compare."""
import numpy as np
import torch

import oracle
from sparse_long_sequence_fwd_b200 import lf_attn, workloads

BF16_MAX_ABS = 2e-2
BF16_REL_RMS = 5e-3
# f16 rounds with unit 2^-11 where bf16 rounds with 2^-8 (inputs, P, output):
# the bf16 bar scaled by 1/8, with some room
F16_MAX_ABS = 4e-3
F16_REL_RMS = 1e-3
F32_MAX_ABS = 1e-5


def run_gpu(w, inp, stream=None):
    dev = {k: (v.cuda() if isinstance(v, torch.Tensor) and k != "dil" else v) for k, v in inp.items()}
    out = lf_attn.fwd(dev["q"], dev["k"], dev["v"], w.r, dil=inp["dil"], global_idx=dev["global_idx"],
                      key_pad_mask=dev["key_pad_mask"], scale=w.softmax_scale, stream=stream,
                      rand_blocks=dev.get("rand_blocks"))
    torch.cuda.synchronize()
    return out


def oracle_full(w, inp, nthreads=0):
    return oracle.fwd(inp["q"], inp["k"], inp["v"], w.r, dil=inp["dil"], global_idx=inp["global_idx"],
                      key_pad_mask=inp["key_pad_mask"], scale=w.softmax_scale, nthreads=nthreads,
                      rand_blocks=inp.get("rand_blocks"))


def oracle_rows(w, inp, rows):
    return oracle.rows(inp["q"], inp["k"], inp["v"], w.r, rows, dil=inp["dil"], global_idx=inp["global_idx"],
                       key_pad_mask=inp["key_pad_mask"], scale=w.softmax_scale)


def compare(w, got, ref):
    """got: torch (any device/dtype), ref: numpy fp64 of the same shape."""
    g = got.detach().double().cpu().numpy()
    assert g.shape == ref.shape
    assert np.all(np.isfinite(g))
    diff = np.abs(g - ref)
    max_abs = float(diff.max()) if diff.size else 0.0
    denom = float(np.sqrt((ref ** 2).sum()))
    rel_rms = float(np.sqrt((diff ** 2).sum()) / denom) if denom > 0 else float(np.sqrt((diff ** 2).sum()))
    if w.dtype == "f32":
        assert max_abs <= F32_MAX_ABS, (max_abs, np.unravel_index(diff.argmax(), diff.shape))
    elif w.dtype == "f16":
        assert max_abs <= F16_MAX_ABS, (max_abs, np.unravel_index(diff.argmax(), diff.shape))
        assert rel_rms <= F16_REL_RMS, rel_rms
    else:
        assert max_abs <= BF16_MAX_ABS, (max_abs, np.unravel_index(diff.argmax(), diff.shape))
        assert rel_rms <= BF16_REL_RMS, rel_rms
    return max_abs, rel_rms


def sample_rows(w, inp, n_random=1500, seed=0):
    """Rows the oracle recomputes one by one at full size: every global row of
    a few heads, sequence ends, 128-row tile boundaries of each residue class,
    padding edges, and seeded random rows."""
    rng = np.random.default_rng(seed)
    T = w.T
    rows = set()
    heads = sorted({0, w.H - 1, w.H // 2} | {h for h in range(w.H) if w.dil[h] != w.dil[0]})
    G = inp["global_idx"]
    for b in range(w.B):
        for h in heads:
            if G is not None:
                for g in set(G[b].tolist()):
                    if 0 <= g < T:
                        rows.add((b, h, g))
            for i in list(range(0, 3)) + list(range(T - 3, T)):
                rows.add((b, h, i))
            dil = int(w.dil[h])
            for c in range(min(dil, T)):
                Tc = (T - c + dil - 1) // dil
                for q0 in range(0, Tc, 128 * 8):
                    for x in (q0 - 1, q0, q0 + 127, q0 + 128):
                        if 0 <= x < Tc:
                            rows.add((b, h, c + dil * x))
        if w.pad_from is not None and w.pad_from[b] is not None:
            p = w.pad_from[b]
            for i in (p - 300, p - 257, p - 1, p, p + 1, p + 256, p + 300):
                if 0 <= i < T:
                    rows.add((b, 0, i))
    for _ in range(n_random):
        rows.add((int(rng.integers(w.B)), int(rng.integers(w.H)), int(rng.integers(T))))
    return np.array(sorted(rows), dtype=np.int32)
