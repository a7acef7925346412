"""lf_attn_fwd_static: the allocation-free entry point.

For callers that cannot call cudaMalloc (graph capture in global mode, a
fixed memory budget, their own pool allocator), lf_attn_fwd_static runs the
same forward on a fixed scratch array compiled into the library.  These
tests call it through the C-ABI, twice in a row, and compare each result
with lf_attn_fwd's on the same inputs, within the tolerances the parity
tests use; they also check that sizes needing more than the fixed scratch
are turned away before anything is launched.  The file name keeps pytest
from collecting it before the other test files.
"""
import numpy as np
import pytest
import torch

from sparse_long_sequence_fwd_b200 import build, lf_attn, workloads

pytestmark = pytest.mark.gpu

SCRATCH_LIMIT = (32 << 20) - 256


@pytest.fixture(scope="module", autouse=True)
def _lib():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    build.build()
    lf_attn.load()
    yield


def _close(w, a, b):
    a64, b64 = a.double().cpu().numpy(), b.double().cpu().numpy()
    diff = np.abs(a64 - b64)
    if w.dtype == "f32":
        assert diff.max() <= 1e-5
    else:
        assert diff.max() <= 2e-2
        assert np.sqrt((diff ** 2).sum() / max((b64 ** 2).sum(), 1e-30)) <= 5e-3


@pytest.mark.parametrize("w", [workloads.TINY, workloads.BASE, workloads.QA,
                               workloads.custom("static_dil", "bf16", 1, 3, 700, 64, 40, dil=[1, 2, 3],
                                                globals_per_b=[[0, 350, 699]], seed=50)],
                         ids=lambda w: w.name)
def test_static_matches_allocating_entry_point_twice(w):
    inp = workloads.make_inputs(w, "cuda")
    kw = dict(dil=inp["dil"], global_idx=inp["global_idx"], key_pad_mask=inp["key_pad_mask"],
              scale=w.softmax_scale)
    ref = lf_attn.fwd(inp["q"], inp["k"], inp["v"], w.r, **kw)
    outs = []
    for _ in range(2):
        out = torch.full_like(inp["q"], float("nan"))
        lf_attn.fwd_static(inp["q"], inp["k"], inp["v"], w.r, out=out, **kw)
        outs.append(out)
    torch.cuda.synchronize()
    for out in outs:
        assert torch.isfinite(out.float()).all()
        _close(w, out, ref)


def test_sizes_beyond_the_scratch_are_rejected_before_launch():
    B, H, T, d, ng = 1, 16, 16384, 64, 4096
    need = lf_attn.workspace_bytes(B, H, T, d, ng, lf_attn.LF_BF16)
    assert need > SCRATCH_LIMIT
    q = torch.zeros(B, H, T, d, dtype=torch.bfloat16, device="cuda")
    out = torch.full_like(q, 3.0)
    g = torch.arange(ng, dtype=torch.int32, device="cuda").reshape(1, ng)
    with pytest.raises(lf_attn.LfAttnError) as e:
        lf_attn.fwd_static(q, q, q, 8, global_idx=g, out=out)
    assert e.value.status == 6
    torch.cuda.synchronize()
    assert torch.all(out == 3.0)  # nothing ran
