"""sv_verify_chain_noalloc (the library's fixed per-device scratch instead of
a caller workspace) against sv_verify_chain, through the C ABI: the same
inputs give the same outputs, on two calls in a row.  Kept in its own file,
collected last."""
import numpy as np
import pytest
import torch

from speculative_decoding_verification_94_b200 import inputs, sv
from tests.parity import assert_close, bitwise_equal

pytestmark = pytest.mark.gpu

DEV = "cuda"


def _chain(fn, x, **kw):
    st = torch.zeros(1, dtype=torch.int32, device=DEV)
    out = fn(x.target.to(DEV), x.draft.to(DEV), x.draft_tokens.to(DEV), x.uniforms.to(DEV),
             x.temperature, device_status=st, **kw)
    torch.cuda.synchronize()
    assert int(st.item()) & sv.SV_DEV_ERROR_MASK == 0
    return out


def test_noalloc_matches_the_workspace_call_twice_in_a_row():
    x = inputs.qwen_chain(B=32, k=3, sigma_d=1.0, seed=11)
    ref = _chain(sv.sv_verify_chain, x)
    for _ in range(2):
        got = _chain(sv.sv_verify_chain_noalloc, x)
        assert torch.equal(got["accepted_len"], ref["accepted_len"])
        assert torch.equal(got["out_tokens"], ref["out_tokens"])


def test_noalloc_fused_kd_matches_twice_in_a_row():
    x = inputs.kd_chain(B=16, k=3, seed=12)
    kd = dict(K=32, reward=x.reward.to(DEV), wmode="group_norm", group=16)
    ref = _chain(sv.sv_verify_chain, x, kd=kd)
    for _ in range(2):
        got = _chain(sv.sv_verify_chain_noalloc, x, kd=kd)
        for key in ("accepted_len", "out_tokens", "topk_idx"):
            assert torch.equal(got[key], ref[key]), key
        for key in ("topk_logp", "lse", "kl", "loss", "total"):
            a, b = got[key].cpu().numpy(), ref[key].cpu().numpy()
            fin = np.isfinite(b)
            assert np.array_equal(np.isnan(a), np.isnan(b)), key
            assert_close(a[fin], b[fin], 1.0, key)
        assert bitwise_equal(got["accepted_len"], ref["accepted_len"])


def test_noalloc_rejects_a_batch_beyond_its_scratch():
    B, k, V = 1024, 3, 151936
    assert sv.sv_verify_chain_workspace_size(B, k, V, 0) > (4 << 20)
    x = inputs.make_chain(B, k, 1024, dtype="bf16", seed=13)  # small tensors, large declared V
    t = torch.zeros(B, k + 1, V, dtype=torch.bfloat16, device=DEV)
    d = torch.zeros(B, k, V, dtype=torch.bfloat16, device=DEV)
    with pytest.raises(sv.SVError) as e:
        sv.sv_verify_chain_noalloc(t, d, x.draft_tokens.to(DEV), x.uniforms.to(DEV), 0.7)
    assert e.value.status == sv.SV_ERR_WORKSPACE


def test_noalloc_scratch_returns_to_zero_after_a_failed_request():
    """A call whose request 1 carries an out-of-range draft token (checked on
    the device, reported in the status word) must leave the fixed scratch as
    zero as a clean call does: the next call matches sv_verify_chain bit for
    bit."""
    x = inputs.qwen_chain(B=16, k=3, sigma_d=1.0, seed=14)
    bad = x.draft_tokens.clone()
    bad[1, 0] = x.V  # outside [0, V)
    st = torch.zeros(1, dtype=torch.int32, device=DEV)
    got = sv.sv_verify_chain_noalloc(x.target.to(DEV), x.draft.to(DEV), bad.to(DEV),
                                     x.uniforms.to(DEV), x.temperature, device_status=st)
    torch.cuda.synchronize()
    assert int(st.item()) & sv.SV_DEV_BAD_TOKEN
    assert got["accepted_len"][1].item() == -1
    assert (got["out_tokens"][1] == -1).all()
    ref = _chain(sv.sv_verify_chain, x)
    for _ in range(2):
        good = _chain(sv.sv_verify_chain_noalloc, x)
        assert torch.equal(good["accepted_len"], ref["accepted_len"])
        assert torch.equal(good["out_tokens"], ref["out_tokens"])
