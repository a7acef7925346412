"""The backward pass (lf_attn_bwd) against the oracle's fp64 gradients
(oracle.bwd, pinned by finite differences in tests/test_oracle_bwd.py) on
the same seeded inputs, every element.

Bar: fp32 inputs, the kernels' fp32 arithmetic: max-abs <= 1e-4 max(1,
max |ref|), rel-RMS <= 1e-5.  16-bit inputs: the oracle takes the rounded
inputs exactly, but D_i = dy_i . y_i uses the forward's output rounded to
the input type, so the forward's 16-bit bar applies, relative to the
gradients' scale: max-abs <= 2e-2 max(1, max |ref|), rel-RMS <= 5e-3."""
import numpy as np
import pytest
import torch

import oracle
from sparse_long_sequence_fwd_b200 import build, lf_attn, workloads

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _lib():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    build.build()
    lf_attn.load()
    yield


CASES = [
    workloads.custom("bwd_f32", "f32", 1, 2, 300, 32, 20, dil=[1, 2], globals_per_b=[[0, 150, 299]],
                     pad_from=[280], seed=91),
    workloads.custom("bwd_bf16", "bf16", 2, 2, 500, 64, 30, dil=[1, 3],
                     globals_per_b=[[5, 5, 400], [0, 250, 499]], pad_from=[None, 450], seed=92),
    workloads.custom("bwd_f16_d128", "f16", 1, 1, 257, 128, 100, seed=93),
    workloads.custom("bwd_bf16_all_padded", "bf16", 2, 1, 64, 64, 5, globals_per_b=[[0], [1]],
                     pad_from=[None, 0], seed=94),
]


@pytest.mark.parametrize("w", CASES, ids=lambda w: w.name)
def test_backward_every_element(w):
    inp = workloads.make_inputs(w)
    g = torch.Generator().manual_seed(w.seed + 1)
    dy = torch.randn(inp["q"].shape, generator=g).to(inp["q"].dtype)
    dev = {k: (v.cuda() if isinstance(v, torch.Tensor) and k != "dil" else v) for k, v in inp.items()}
    y = lf_attn.fwd(dev["q"], dev["k"], dev["v"], w.r, dil=inp["dil"], global_idx=dev["global_idx"],
                    key_pad_mask=dev["key_pad_mask"], scale=w.softmax_scale)
    got = lf_attn.bwd(dev["q"], dev["k"], dev["v"], y, dy.cuda(), w.r, dil=inp["dil"], global_idx=dev["global_idx"],
                      key_pad_mask=dev["key_pad_mask"], scale=w.softmax_scale)
    torch.cuda.synchronize()
    ref = oracle.bwd(inp["q"], inp["k"], inp["v"], dy, w.r, dil=inp["dil"], global_idx=inp["global_idx"],
                     key_pad_mask=inp["key_pad_mask"], scale=w.softmax_scale)
    for name, a, b in zip(("dq", "dk", "dv"), got, ref):
        a = a.double().cpu().numpy()
        assert np.all(np.isfinite(a)), name
        diff = np.abs(a - b)
        top = max(1.0, float(np.abs(b).max()))
        rel_rms = float(np.sqrt((diff ** 2).sum() / max((b ** 2).sum(), 1e-300)))
        if w.dtype == "f32":
            assert diff.max() <= 1e-4 * top, (name, diff.max())
            assert rel_rms <= 1e-5 or np.sqrt((b ** 2).sum()) == 0, (name, rel_rms)
        else:
            assert diff.max() <= 2e-2 * top, (name, diff.max())
            assert rel_rms <= 5e-3 or np.sqrt((b ** 2).sum()) == 0, (name, rel_rms)
