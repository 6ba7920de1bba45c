"""A bounded device wait that runs out.

The persistent chain kernel's test hook makes the warp that reduces request 0's first
slice wait on a barrier nothing arrives on, under a short wait limit: the wait
gives up, the call returns, reports SV_DEV_TIMEOUT, fails request 0 only
(accepted length -1, tokens -1), leaves the workspace all zero, and the next
call is correct.  No GPU fault or hang is involved: the wait is bounded by
the kernel's own time limit."""
import numpy as np
import pytest
import torch

from oracle import oracle as O
from speculative_decoding_verification_94_b200 import inputs, sv
from tests.parity import assert_chain_match

pytestmark = pytest.mark.gpu
DEV = "cuda"


def _run(x, st):
    return sv.sv_verify_chain(x.target.to(DEV), x.draft.to(DEV), x.draft_tokens.to(DEV),
                              x.uniforms.to(DEV), x.temperature, device_status=st)


def test_bounded_wait_runs_out_and_reports():
    x = inputs.qwen_chain(B=8, k=3, sigma_d=1.0, seed=21)
    ref = O.verify_chain(x.target, x.draft, x.draft_tokens, x.uniforms, x.temperature)
    st = torch.zeros(1, dtype=torch.int32, device=DEV)
    with sv.knobs(persistent=1, wait_ns=20_000_000, stall=1):  # 20 ms limit; the stalled wait gives up at 5 ms
        got = _run(x, st)
        torch.cuda.synchronize()
    word = int(st.item())
    assert word & sv.SV_DEV_TIMEOUT, hex(word)
    assert sv.sv_device_status_check(word) == sv.SV_ERR_TIMEOUT
    acc = got["accepted_len"].cpu().numpy()
    out = got["out_tokens"].cpu().numpy()
    assert acc[0] == -1 and (out[0] == -1).all()
    # every other request is unaffected
    sub = {k: v[1:] for k, v in ref.items() if isinstance(v, np.ndarray) and v.shape[:1] == (8,)}
    assert_chain_match({"accepted_len": got["accepted_len"][1:], "out_tokens": got["out_tokens"][1:]},
                       sub, x.uniforms.numpy()[1:], x.temperature, x.k)
    ws = sv._WS[torch.cuda.current_device()]
    assert int(torch.count_nonzero(ws)) == 0
    # the next call, without the hook, is whole
    st.zero_()
    again = _run(x, st)
    torch.cuda.synchronize()
    assert int(st.item()) & sv.SV_DEV_ERROR_MASK == 0
    assert np.array_equal(again["accepted_len"].cpu().numpy(), ref["accepted_len"])
    assert np.array_equal(again["out_tokens"].cpu().numpy(), ref["out_tokens"])
    assert int(torch.count_nonzero(ws)) == 0
