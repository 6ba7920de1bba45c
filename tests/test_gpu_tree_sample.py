"""Sampling tree verification (sv_verify_tree_sample) against the float64
oracle, and its losslessness on the GPU.

Integers must match exactly except for requests whose decisions lie near a
boundary in the oracle's exact arithmetic: a child test with
|u - r(x)/q(x)| < 1e-6, or a draw within 1e-6 of an inverse-CDF step (the
chain's window).  The kernel forms the row statistics, p(x), q(x), the
residual max(0, p - sigma q) and its mass in float64, so the running residual
carries float64 rounding although p - sigma q cancels where the rows agree;
flagged requests are counted and checked for well-formed outputs only."""
import numpy as np
import pytest
import torch

from oracle import oracle as O
from speculative_decoding_verification_94_b200 import inputs, sv

pytestmark = pytest.mark.gpu

DEV = "cuda"
WINDOW = 1e-6


def _run(x, draft=None, kind="logits", status=None):
    d = x.draft if draft is None else draft
    return sv.sv_verify_tree_sample(x.target.to(DEV), d.to(DEV), x.node_tokens.to(DEV),
                                    x.parents.to(DEV), x.uniforms.to(DEV), x.temperature,
                                    x.max_depth, draft_kind=kind, device_status=status)


def _compare(got, ref, max_flag_frac=0.1):
    acc = got["accepted_len"].cpu().numpy()
    out = got["out_tokens"].cpu().numpy()
    nodes = got["accepted_nodes"].cpu().numpy()
    flags = (ref["test_margin"] < WINDOW) | (ref["cdf_margin"] < WINDOW)
    same = ((acc == ref["accepted_len"]) & (out == ref["out_tokens"]).all(1) &
            (nodes == ref["accepted_nodes"]).all(1))
    bad = np.nonzero(~same & ~flags)[0]
    assert bad.size == 0, (
        f"{bad.size} unflagged mismatches, first b={bad[0]}: gpu {acc[bad[0]]} {out[bad[0]]} "
        f"{nodes[bad[0]]}; oracle {ref['accepted_len'][bad[0]]} {ref['out_tokens'][bad[0]]} "
        f"{ref['accepted_nodes'][bad[0]]}")
    for b in np.nonzero(flags)[0]:
        a = acc[b]
        assert a >= 0 and out[b, a] >= 0 and (out[b, a + 1:] == -1).all()
        assert nodes[b, 0] == 0
    assert flags.mean() <= max_flag_frac, f"{flags.sum()} of {flags.size} flagged"
    return dict(flagged=int(flags.sum()), mismatched_flagged=int((~same & flags).sum()))


def test_tree_sample_full_vocabulary():
    """EAGLE-shaped trees (s, t, n) = (5, 8, 32) at the Qwen vocabulary."""
    x = inputs.make_tree_sample(B=16, seed=3)
    st = torch.zeros(1, dtype=torch.int32, device=DEV)
    got = _run(x, status=st)
    torch.cuda.synchronize()
    assert int(st.item()) & sv.SV_DEV_ERROR_MASK == 0
    ref = O.tree_sample(x.target, x.draft, x.node_tokens, x.parents, x.uniforms, x.temperature,
                        x.max_depth)
    r = _compare(got, ref, max_flag_frac=0.25)
    print("tree sample full V", r, np.bincount(ref["accepted_len"]), ref["n_tests"].tolist())
    assert ref["n_tests"].max() >= 2  # residual passes were exercised


@pytest.mark.parametrize("ctas", ["1", "2", "5", "16"])
def test_tree_sample_cluster_sizes(ctas):
    with sv.knobs(cluster_ctas=int(ctas)):
        _tree_cluster_case()


def _tree_cluster_case():
    x = inputs.make_tree_sample(B=24, V=20000, depth_counts=(4, 4, 3), branching=4,
                                sigma_d=0.7, temperature=0.9, seed=5)
    st = torch.zeros(1, dtype=torch.int32, device=DEV)
    got = _run(x, status=st)
    torch.cuda.synchronize()
    assert int(st.item()) & sv.SV_DEV_ERROR_MASK == 0
    ref = O.tree_sample(x.target, x.draft, x.node_tokens, x.parents, x.uniforms, x.temperature,
                        x.max_depth)
    _compare(got, ref, max_flag_frac=0.25)


@pytest.mark.parametrize("dtype,kind", [("f32", "logits"), ("bf16", "logits"),
                                        ("f32", "probs")])
def test_tree_sample_many_small_trees(dtype, kind):
    x = inputs.make_tree_sample(B=3000, V=203, depth_counts=(4, 4, 4, 2), branching=4,
                                dtype=dtype, model="gauss", sigma_t=2.0, sigma_d=0.8,
                                temperature=1.0, seed=11)
    draft = x.draft
    okind = O.DRAFT_LOGITS
    if kind == "probs":
        draft = torch.softmax(x.draft.double() / x.temperature, dim=-1).float()
        okind = O.DRAFT_PROBS
    st = torch.zeros(1, dtype=torch.int32, device=DEV)
    got = _run(x, draft, kind, status=st)
    torch.cuda.synchronize()
    assert int(st.item()) & sv.SV_DEV_ERROR_MASK == 0
    ref = O.tree_sample(x.target, draft, x.node_tokens, x.parents, x.uniforms, x.temperature,
                        x.max_depth, draft_kind=okind)
    r = _compare(got, ref)
    print("small trees", dtype, kind, r, np.bincount(ref["accepted_len"]))
    assert len(set(ref["accepted_len"].tolist())) >= 4


def test_tree_sample_gpu_losslessness():
    """Depth-2 context-consistent trees, children drawn from the draft rows:
    the emitted token at each position follows the target row of its
    context (chi-square over 10^6 trees on the GPU)."""
    import scipy.stats
    rng = np.random.default_rng(29)
    V, m1, m2, B = 5, 3, 2, 1_000_000
    p0 = rng.dirichlet(np.full(V, 0.8))
    p1 = rng.dirichlet(np.full(V, 0.8), size=V)
    p2 = rng.dirichlet(np.full(V, 0.8), size=(V, V))
    q0 = rng.dirichlet(np.full(V, 0.8))
    q1 = rng.dirichlet(np.full(V, 0.8), size=V)
    n = 1 + m1 + m1 * m2
    par = np.full((B, n), -1, np.int32)
    par[:, 1:1 + m1] = 0
    for i in range(m1):
        par[:, 1 + m1 + i * m2:1 + m1 + (i + 1) * m2] = 1 + i
    tok = np.zeros((B, n), np.int32)
    c0 = np.cumsum(q0)
    tok[:, 1:1 + m1] = np.minimum((rng.random((B, m1))[:, :, None] > c0).sum(-1), V - 1)
    c1 = np.cumsum(q1, axis=1)
    for i in range(m1):
        t1 = tok[:, 1 + i]
        d = (rng.random((B, m2))[:, :, None] > c1[t1][:, None, :]).sum(-1)
        tok[:, 1 + m1 + i * m2:1 + m1 + (i + 1) * m2] = np.minimum(d, V - 1)
    logp = np.zeros((B, n, V), np.float32)
    qd = np.zeros((B, n, V), np.float32)
    logp[:, 0] = np.log(p0)
    qd[:, 0] = q0
    for i in range(m1):
        t1 = tok[:, 1 + i]
        logp[:, 1 + i] = np.log(p1[t1])
        qd[:, 1 + i] = q1[t1]
        for j in range(m2):
            c = 1 + m1 + i * m2 + j
            logp[:, c] = np.log(p2[t1, tok[:, c]])
            qd[:, c] = q0
    u = inputs.uniforms24(np.random.default_rng(30), (B, n))
    st = torch.zeros(1, dtype=torch.int32, device=DEV)
    got = sv.sv_verify_tree_sample(torch.from_numpy(logp).to(DEV), torch.from_numpy(qd).to(DEV),
                                   torch.from_numpy(tok).to(DEV), torch.from_numpy(par).to(DEV),
                                   torch.from_numpy(u).to(DEV), 1.0, 2, draft_kind="probs",
                                   device_status=st)
    torch.cuda.synchronize()
    assert int(st.item()) & sv.SV_DEV_ERROR_MASK == 0
    acc = got["accepted_len"].cpu().numpy()
    out = got["out_tokens"].cpu().numpy()

    def sm(z):
        z = z.astype(np.float32).astype(np.float64)
        e = np.exp(z - z.max(-1, keepdims=True))
        return e / e.sum(-1, keepdims=True)

    P0, P1, P2 = sm(np.log(p0)), sm(np.log(p1)), sm(np.log(p2))
    pv = [scipy.stats.chisquare(np.bincount(out[:, 0], minlength=V), P0 * B).pvalue]
    for t in range(V):
        sel = (acc >= 1) & (out[:, 0] == t)
        if sel.sum() >= 1000:
            pv.append(scipy.stats.chisquare(np.bincount(out[sel, 1], minlength=V),
                                            P1[t] * sel.sum()).pvalue)
        for t2 in range(V):
            sel2 = sel & (acc >= 2) & (out[:, 1] == t2)
            if sel2.sum() >= 1000:
                pv.append(scipy.stats.chisquare(np.bincount(out[sel2, 2], minlength=V),
                                                P2[t, t2] * sel2.sum()).pvalue)
    assert len(pv) > 10
    assert min(pv) > 1e-4, pv


def test_tree_sample_edge_cases():
    # a lone root: one draw from p_root
    x = inputs.make_tree_sample(B=64, V=1001, depth_counts=(), seed=8)
    got = _run(x)
    ref = O.tree_sample(x.target, x.draft, x.node_tokens, x.parents, x.uniforms, x.temperature, 0)
    torch.cuda.synchronize()
    _compare(got, ref, max_flag_frac=0.1)
    assert (got["accepted_len"].cpu().numpy() == 0).all()
    # malformed trees, bad tokens and rows without a finite value fail only their request
    x = inputs.make_tree_sample(B=4, V=4099, depth_counts=(3, 2), branching=3, seed=9)
    par = x.parents.clone()
    tok = x.node_tokens.clone()
    tgt = x.target.clone()
    par[0, 2] = 2            # not a parent before the node
    tok[1, 3] = 4099         # token outside [0, V)
    tgt[2, 0] = float("-inf")  # the root's target row has no finite value
    st = torch.zeros(1, dtype=torch.int32, device=DEV)
    got = sv.sv_verify_tree_sample(tgt.to(DEV), x.draft.to(DEV), tok.to(DEV), par.to(DEV),
                                   x.uniforms.to(DEV), x.temperature, x.max_depth,
                                   device_status=st)
    torch.cuda.synchronize()
    s = int(st.item())
    assert s & sv.SV_DEV_BAD_TREE and s & sv.SV_DEV_BAD_TOKEN and s & sv.SV_DEV_NO_FINITE
    acc = got["accepted_len"].cpu().numpy()
    assert (acc[:3] == -1).all()
    assert (got["out_tokens"].cpu().numpy()[:3] == -1).all()
    ref = O.tree_sample(x.target[3:], x.draft[3:], x.node_tokens[3:], x.parents[3:],
                        x.uniforms[3:], x.temperature, x.max_depth)
    assert acc[3] == ref["accepted_len"][0] or ref["cdf_margin"][0] < WINDOW
