"""Kernel marks (SV_KNOB_KERNEL_MARKS) through the C ABI: a marked chain call
reports one streaming pass and one finishing kernel (two-kernel path) or one
persistent launch, each with a positive device time, and reading the marks
starts a new count."""
import pytest
import torch

from speculative_decoding_verification_94_b200 import inputs, sv

pytestmark = pytest.mark.gpu
DEV = "cuda"


def _call(x):
    return sv.sv_verify_chain(x.target.to(DEV), x.draft.to(DEV), x.draft_tokens.to(DEV),
                              x.uniforms.to(DEV), x.temperature)


@pytest.mark.parametrize("path,kinds", [({}, ["stream", "finish"]),
                                        (dict(persistent=1), ["chain"])])
def test_marked_call_reports_its_launches(path, kinds):
    x = inputs.make_chain(4, 3, 4099, dtype="bf16", sigma_d=1.0, temperature=0.7, seed=31)
    sv.sv_kernel_times()  # drop earlier marks
    with sv.knobs(kernel_marks=1, **path):
        _call(x)
        torch.cuda.synchronize()
    marks = sv.sv_kernel_times()
    assert [m[0] for m in marks] == kinds
    assert all(0.0 < us < 1e6 for _, us in marks)
    assert sv.sv_kernel_times() == []
    # unmarked calls add nothing
    _call(x)
    torch.cuda.synchronize()
    assert sv.sv_kernel_times() == []


def test_marks_inside_a_captured_graph():
    x = inputs.make_chain(4, 3, 4099, dtype="bf16", sigma_d=1.0, temperature=0.7, seed=32)
    t, d, tok, u = (x.target.to(DEV), x.draft.to(DEV), x.draft_tokens.to(DEV), x.uniforms.to(DEV))
    with sv.knobs(kernel_marks=1):
        sv.sv_verify_chain(t, d, tok, u, 0.7)  # the events exist before capture
        torch.cuda.synchronize()
        sv.sv_kernel_times()
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g):
            for _ in range(3):
                sv.sv_verify_chain(t, d, tok, u, 0.7)
    g.replay()
    torch.cuda.synchronize()
    marks = sv.sv_kernel_times()
    assert [m[0] for m in marks] == ["stream", "finish"] * 3
    assert all(us > 0.0 for _, us in marks)
