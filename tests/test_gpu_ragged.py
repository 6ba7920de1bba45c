"""Ragged batches (sv_verify_chain_ragged) against the float64 oracle: each
request verifies its own number of drafts k_b <= k, idle requests emit
nothing.  The GPU gets inputs whose unused entries are poisoned (rows of
-inf, draft tokens outside [0, V)): if any of them were read, the call would
report SV_DEV_NO_FINITE or SV_DEV_BAD_TOKEN or give different results; the
oracle gets the clean inputs."""
import numpy as np
import pytest
import torch

from oracle import oracle as O
from speculative_decoding_verification_94_b200 import inputs, sv
from tests.parity import assert_chain_match, assert_close

pytestmark = pytest.mark.gpu

DEV = "cuda"


def _lengths(B, k, seed, idle_frac=0.15):
    rng = np.random.default_rng(seed)
    klen = rng.integers(0, k + 1, B).astype(np.int32)
    act = (rng.random(B) >= idle_frac).astype(np.int32)
    n = min(B, k + 1)
    klen[:n] = np.arange(n)  # every length occurs
    act[:n] = 1
    if B > k + 1:
        act[k + 1] = 0
    return klen, act


def _poisoned(x, klen, act):
    tgt = x.target.clone()
    dft = x.draft.clone() if x.draft is not None else None
    tok = x.draft_tokens.clone()
    for b in range(x.B):
        lo_t = int(klen[b]) + 1 if act[b] else 0
        lo_d = int(klen[b]) if act[b] else 0
        tgt[b, lo_t:] = float("-inf")
        if dft is not None:
            dft[b, lo_d:] = float("-inf")
        tok[b, lo_d:] = x.V + 7
    return inputs.ChainInputs(tgt, dft, tok, x.uniforms, x.reward, x.temperature, x.draft_kind)


def _run(x, klen, act, kd=None, status=None):
    return sv.sv_verify_chain_ragged(
        x.target.to(DEV), x.draft.to(DEV) if x.draft is not None else None,
        x.draft_tokens.to(DEV), x.uniforms.to(DEV) if x.uniforms is not None else None,
        x.temperature, draft_len=torch.from_numpy(klen).to(DEV),
        active=torch.from_numpy(act).to(DEV), draft_kind=x.draft_kind, kd=kd,
        device_status=status)


def _check_idle(got, act):
    acc = got["accepted_len"].cpu().numpy()
    out = got["out_tokens"].cpu().numpy()
    assert (acc[act == 0] == 0).all()
    assert (out[act == 0] == -1).all()


PATHS = {"persistent": dict(persistent=1), "persistent-order2": dict(persistent=1, order=2),
         "two-kernel-static": dict(stream_count=1), "two-kernel-dynamic": dict(stream_count=2)}


@pytest.fixture(params=list(PATHS))
def path(request):
    with sv.knobs(**PATHS[request.param]):
        yield request.param


@pytest.mark.parametrize("k,sigma", [(3, 1.0), (5, 0.5)])
def test_ragged_sampling_chain(path, k, sigma):
    x = inputs.qwen_chain(B=32, k=k, sigma_d=sigma, seed=40 + k)
    klen, act = _lengths(x.B, k, seed=k)
    st = torch.zeros(1, dtype=torch.int32, device=DEV)
    got = _run(_poisoned(x, klen, act), klen, act, status=st)
    torch.cuda.synchronize()
    assert int(st.item()) & sv.SV_DEV_ERROR_MASK == 0
    ref = O.verify_chain(x.target, x.draft, x.draft_tokens, x.uniforms, x.temperature,
                         draft_len=klen, active=act)
    assert_chain_match(got, ref, x.uniforms.numpy(), x.temperature, k, max_flag_frac=0.1)
    _check_idle(got, act)
    assert (got["accepted_len"].cpu().numpy() <= klen).all()
    ws = sv._WS[torch.cuda.current_device()]
    assert int(torch.count_nonzero(ws)) == 0


def test_ragged_greedy_chain(path):
    x = inputs.make_chain(40, 4, 70001, dtype="bf16", sigma_d=0.3, temperature=0.0, seed=12)
    klen, act = _lengths(x.B, x.k, seed=3)
    st = torch.zeros(1, dtype=torch.int32, device=DEV)
    got = _run(_poisoned(x, klen, act), klen, act, status=st)
    torch.cuda.synchronize()
    assert int(st.item()) & sv.SV_DEV_ERROR_MASK == 0
    ref = O.verify_chain(x.target, None, x.draft_tokens, None, 0.0, draft_len=klen, active=act)
    assert np.array_equal(got["accepted_len"].cpu().numpy(), ref["accepted_len"])
    assert np.array_equal(got["out_tokens"].cpu().numpy(), ref["out_tokens"])
    assert len(set(ref["accepted_len"][act == 1].tolist())) > 1


def test_ragged_fused_kd(path):
    """Fused KD on a ragged batch: rows 0..n of each active request defined,
    no KL for the bonus row k_b, idle requests empty, loss with n < k_b for
    the first-rejected-position rule."""
    x = inputs.kd_chain(B=48, k=4, seed=3)
    klen, act = _lengths(x.B, x.k, seed=11)
    st = torch.zeros(1, dtype=torch.int32, device=DEV)
    kd = dict(K=32, reward=x.reward.to(DEV), wmode="group_norm", group=16, positions=1)
    got = _run(_poisoned(x, klen, act), klen, act, kd=kd, status=st)
    torch.cuda.synchronize()
    assert int(st.item()) & sv.SV_DEV_ERROR_MASK == 0
    ref = O.verify_kd(x.target, x.draft, x.draft_tokens, x.uniforms, x.reward, x.temperature, 32,
                      mode=O.W_GROUP_NORM, group=16, positions=1, draft_len=klen, active=act)
    assert_chain_match(got, ref, x.uniforms.numpy(), x.temperature, x.k, max_flag_frac=0.1)
    _check_idle(got, act)
    acc = got["accepted_len"].cpu().numpy()
    on = act == 1
    tmask = (np.arange(x.k + 1)[None, :] <= acc[:, None]) & on[:, None]
    dmask = (np.arange(x.k)[None, :] <= acc[:, None]) & \
            (np.arange(x.k)[None, :] < klen[:, None]) & on[:, None]
    idx = got["topk_idx"].cpu().numpy()
    assert np.array_equal(idx[tmask], ref["topk_idx"][tmask])
    assert (idx[~tmask] == -1).all()
    lp = got["topk_logp"].cpu().numpy()
    assert_close(lp[tmask], ref["topk_logp"][tmask], 1.0, "topk_logp")
    assert np.isnan(lp[~tmask]).all()
    lse = got["lse"].cpu().numpy()
    assert_close(lse[tmask], ref["lse"][tmask], 1.0, "lse")
    assert np.isnan(lse[~tmask]).all()
    kl = got["kl"].cpu().numpy()
    assert_close(kl[dmask], ref["kl"][dmask], ref["scale"][dmask], "kl")
    assert np.isnan(kl[~dmask]).all()
    rl = O.reward_loss(ref["kl"], acc, x.reward.numpy().astype(np.float64), mode=O.W_GROUP_NORM,
                       group=16, positions=1, draft_len=klen, active=act)
    m = np.where(acc < klen, acc + 1, acc) * on
    mag = np.array([abs(rl["w"][b]) * ref["scale"][b, :m[b]].sum() for b in range(x.B)])
    assert_close(got["loss"].cpu().numpy(), rl["loss"], mag, "loss")
    assert_close(got["total"].cpu().numpy(), [rl["total"]], [mag.sum()], "total")
    assert (got["loss"].cpu().numpy()[~on] == 0).all()
    ws = sv._WS[torch.cuda.current_device()]
    assert int(torch.count_nonzero(ws)) == 0


def test_ragged_full_lengths_equal_the_padded_call():
    """draft_len = k and every request active: bit-identical to sv_verify_chain."""
    x = inputs.qwen_chain(B=16, k=3, sigma_d=1.0, seed=2)
    klen = np.full(x.B, x.k, np.int32)
    act = np.ones(x.B, np.int32)
    kd = dict(K=32, reward=x.reward.to(DEV))
    a = _run(x, klen, act, kd=kd)
    b = sv.sv_verify_chain(x.target.to(DEV), x.draft.to(DEV), x.draft_tokens.to(DEV),
                           x.uniforms.to(DEV), x.temperature, kd=kd)
    torch.cuda.synchronize()
    for key in ("accepted_len", "out_tokens", "topk_idx"):
        assert torch.equal(a[key], b[key]), key
    for key in ("topk_logp", "lse", "kl", "loss", "total"):
        assert torch.equal(torch.nan_to_num(a[key], nan=7.0), torch.nan_to_num(b[key], nan=7.0)), key


def test_ragged_invalid_length_and_all_idle():
    """A draft_len outside [0, k] fails only its request (SV_DEV_BAD_LEN);
    a batch with every request idle reads nothing and leaves the workspace
    zero."""
    x = inputs.make_chain(6, 3, 5000, dtype="bf16", sigma_d=1.0, temperature=0.9, seed=4)
    klen = np.array([3, 4, 1, -1, 0, 2], np.int32)
    act = np.ones(6, np.int32)
    st = torch.zeros(1, dtype=torch.int32, device=DEV)
    got = _run(x, klen, act, status=st)
    torch.cuda.synchronize()
    assert int(st.item()) & sv.SV_DEV_BAD_LEN
    acc = got["accepted_len"].cpu().numpy()
    out = got["out_tokens"].cpu().numpy()
    assert acc[1] == -1 and acc[3] == -1 and (out[[1, 3]] == -1).all()
    good = np.array([0, 2, 4, 5])
    ref = O.verify_chain(x.target[good], x.draft[good], x.draft_tokens[good], x.uniforms[good],
                         x.temperature, draft_len=klen[good])
    assert np.array_equal(acc[good], ref["accepted_len"])
    assert np.array_equal(out[good], ref["out_tokens"])
    idle = np.zeros(6, np.int32)
    st.zero_()
    got = _run(_poisoned(x, klen * 0, idle), klen * 0, idle, status=st)
    torch.cuda.synchronize()
    assert int(st.item()) == 0
    _check_idle(got, idle)
    ws = sv._WS[torch.cuda.current_device()]
    assert int(torch.count_nonzero(ws)) == 0
