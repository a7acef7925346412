"""lf_attn_fwd_static: the allocation-free entry point.

For callers that cannot call cudaMalloc (graph capture in global mode, a
fixed memory budget, their own pool allocator), lf_attn_fwd_static runs the
same forward on a fixed scratch array compiled into the library.  These
tests call it through the C-ABI, twice in a row, and compare each result
with lf_attn_fwd's on the same inputs: the two entry points run the same
kernels on the same inputs, so the outputs must be equal bit for bit.  One
case is also compared with the fp64 oracle directly, within the parity
tests' tolerances.  They also check that sizes needing more than the fixed
scratch are turned away before anything is launched.  The file name keeps
pytest from collecting it before the other test files.
"""
import pytest
import torch

from sparse_long_sequence_fwd_b200 import build, lf_attn, workloads
from tests import parity

pytestmark = pytest.mark.gpu

SCRATCH_LIMIT = (32 << 20) - 256


@pytest.fixture(scope="module", autouse=True)
def _lib():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    build.build()
    lf_attn.load()
    yield


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
        assert torch.equal(out, ref)


def test_static_matches_the_oracle():
    """Two calls in a row on a multi-tile case with dilation, globals and
    padding, each compared with the fp64 oracle on every element."""
    w = workloads.custom("static_oracle", "bf16", 2, 3, 900, 64, 70, dil=[1, 2, 3],
                         globals_per_b=[[0, 450, 450], [3, 3, 899]], pad_from=[None, 800], seed=51)
    cpu = workloads.make_inputs(w)
    inp = workloads.make_inputs(w, "cuda")
    ref = parity.oracle_full(w, cpu)
    for _ in range(2):
        out = torch.full_like(inp["q"], float("nan"))
        lf_attn.fwd_static(inp["q"], inp["k"], inp["v"], w.r, dil=inp["dil"], global_idx=inp["global_idx"],
                           key_pad_mask=inp["key_pad_mask"], scale=w.softmax_scale, out=out)
        torch.cuda.synchronize()
        parity.compare(w, out, ref)


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


def test_static_runs_inside_a_global_mode_graph_capture():
    """After one call that sets the device up, lf_attn_fwd_static is captured
    into a CUDA graph in global capture mode (where any allocation would
    fail the capture); the replayed graph gives lf_attn_fwd's output."""
    w = workloads.custom("static_graph", "bf16", 1, 4, 1500, 64, 60, dil=[1, 2, 1, 2],
                         globals_per_b=[[3, 700, 1499]], pad_from=[1400], seed=52)
    inp = workloads.make_inputs(w, "cuda")
    kw = dict(dil=inp["dil"], global_idx=inp["global_idx"], key_pad_mask=inp["key_pad_mask"],
              scale=w.softmax_scale)
    ref = lf_attn.fwd(inp["q"], inp["k"], inp["v"], w.r, **kw)
    s = torch.cuda.Stream()
    out = torch.empty_like(inp["q"])
    lf_attn.fwd_static(inp["q"], inp["k"], inp["v"], w.r, out=out, stream=s, **kw)
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=s, capture_error_mode="global"):
        lf_attn.fwd_static(inp["q"], inp["k"], inp["v"], w.r, out=out, stream=s, **kw)
    out.fill_(float("nan"))
    torch.cuda.synchronize()
    g.replay()
    torch.cuda.synchronize()
    assert torch.equal(out, ref)
