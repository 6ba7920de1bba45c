"""Pins of the float64 oracle against what the pages and the mathematics fix.

None of these tests re-derives the oracle's own formulas: each checks it
against a theorem (losslessness of speculative sampling; the acceptance
probability sum_x min(p, q)), a special case with a closed form, brute force
on tiny inputs, an independent library routine (torch / scipy / numpy), or a
worked example printed on the pages (tests/golden).
"""
import json
import math
import os

import numpy as np
import pytest
import scipy.special
import scipy.stats
import torch

from speculative_decoding_verification_94_b200 import inputs

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _kind(o, x):
    return o.DRAFT_PROBS if x.draft_kind == "probs" else o.DRAFT_LOGITS


# --------------------------------------------------------------------------
# Softmax normalisation: an independent library routine.
# --------------------------------------------------------------------------
@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("T", [0.7, 1.0, 2.5])
def test_softmax_matches_torch_float64(oracle, dtype, T):
    x = inputs.make_chain(2, 1, 3001, dtype=dtype, temperature=T, seed=3)
    z = x.target
    got = oracle.softmax(z, T)
    Tf = float(np.float32(T))
    ref = torch.softmax(z.double() / Tf, dim=-1).numpy()
    lz = torch.logsumexp(z.double() / Tf, dim=-1).numpy()
    assert np.allclose(got["p"], ref, rtol=1e-12, atol=1e-300)
    assert np.allclose(got["log_partition"], lz, rtol=1e-13, atol=0)


# --------------------------------------------------------------------------
# Acceptance rule: special cases with closed forms.
# --------------------------------------------------------------------------
@pytest.mark.parametrize("dtype,T", [("f32", 1.0), ("bf16", 0.7), ("bf16", 1.3)])
def test_identical_draft_accepts_every_token(oracle, dtype, T):
    """q == p: min(1, p/q) = 1, so all k drafts are accepted."""
    x = inputs.make_chain(16, 4, 777, dtype=dtype, sigma_d=0.0, temperature=T, seed=5)
    assert torch.equal(x.target[:, :4], x.draft)
    r = oracle.verify_chain(x.target, x.draft, x.draft_tokens, x.uniforms, T)
    assert (r["accepted_len"] == 4).all()
    assert (r["out_tokens"][:, :4] == x.draft_tokens.numpy()).all()
    assert (r["out_tokens"][:, 4] >= 0).all()


def test_disjoint_support_rejects_first_and_resamples_target(oracle):
    """q disjoint from p: p(x) = 0 for every draft, so position 0 always
    rejects (even for u = 0) and the residual max(0, p - q) is p itself: the
    emitted token is the inverse-CDF draw from p_0 (numpy searchsorted)."""
    V, k, B = 64, 3, 256
    rng = np.random.default_rng(0)
    zt = rng.normal(0, 2, (k + 1, V)).astype(np.float32)
    zd = rng.normal(0, 2, (k, V)).astype(np.float32)
    zt[:, 1::2] = -np.inf
    zd[:, 0::2] = -np.inf
    x = inputs.make_chain_fixed(B, zt, zd, draft_kind="logits", temperature=1.0, seed=1)
    x.uniforms[:4, 0] = 0.0
    r = oracle.verify_chain(x.target, x.draft, x.draft_tokens, x.uniforms, 1.0)
    assert (r["accepted_len"] == 0).all()
    p0 = torch.softmax(torch.from_numpy(zt[0]).double(), -1).numpy()
    cdf = np.cumsum(p0)
    expect = np.searchsorted(cdf / cdf[-1], x.uniforms[:, k].double().numpy(), side="right")
    assert (r["out_tokens"][:, 0] == expect).all()
    assert (r["out_tokens"][:, 0] % 2 == 0).all()
    assert (r["out_tokens"][:, 1:] == -1).all()


def test_two_token_disjoint_closed_form(oracle):
    """V=2, p=(1,0), q=(0,1): the draft is token 1, always rejected, and the
    residual puts all mass on token 0."""
    zt = np.array([[0.0, -np.inf]] * 2, np.float32)
    zd = np.array([[-np.inf, 0.0]], np.float32)
    x = inputs.make_chain_fixed(64, zt, zd, draft_kind="logits", seed=2)
    r = oracle.verify_chain(x.target, x.draft, x.draft_tokens, x.uniforms, 1.0)
    assert (x.draft_tokens.numpy() == 1).all()
    assert (r["accepted_len"] == 0).all() and (r["out_tokens"][:, 0] == 0).all()


def test_acceptance_fraction_on_a_uniform_grid(oracle):
    """With u on the grid m/M, the number of accepted draws of a fixed token x
    is #{m : m/M < p(x)/q(x)} = ceil(M p/q) when p/q < 1: the rule is
    'accept with probability min(1, p/q)', checked without sampling noise."""
    V, M = 10, 4096
    zt = np.linspace(-1, 1, V, dtype=np.float32)[None].repeat(2, 0)
    q = np.linspace(2, 0.5, V) ** 2
    q = (q / q.sum()).astype(np.float32)[None]
    x = inputs.make_chain_fixed(M, zt, q, draft_kind="probs", seed=3)
    x.draft_tokens[:] = 0
    x.uniforms[:, 0] = torch.arange(M, dtype=torch.float32) / M
    r = oracle.verify_chain(x.target, x.draft, x.draft_tokens, x.uniforms, 1.0,
                            draft_kind=oracle.DRAFT_PROBS)
    p = torch.softmax(torch.from_numpy(zt[0]).double(), -1).numpy()
    ratio = p[0] / float(q[0, 0])
    assert ratio < 1
    assert int((r["accepted_len"] == 1).sum()) == math.ceil(M * ratio)


# --------------------------------------------------------------------------
# Losslessness (Leviathan et al.): the emitted token at every position is
# distributed as the target row, whatever the draft.  Monte-Carlo chi-square.
# --------------------------------------------------------------------------
def _chain_mc(oracle, draft_kind, T, seed, plant=0, B=200_000, V=8, k=3):
    rng = np.random.default_rng(100 + seed)
    zt = rng.normal(0, 1.5, (k + 1, V)).astype(np.float32)
    if draft_kind == "probs":
        d = rng.dirichlet(np.full(V, 0.7), size=k).astype(np.float32)
        q = d.astype(np.float64)
    else:
        d = (zt[:k] + rng.normal(0, 1.0, (k, V))).astype(np.float32)
        q = torch.softmax(torch.from_numpy(d).double() / float(np.float32(T)), -1).numpy()
    x = inputs.make_chain_fixed(B, zt, d, draft_kind=draft_kind, temperature=T, seed=seed)
    r = oracle.verify_chain(x.target, x.draft, x.draft_tokens, x.uniforms, T,
                            draft_kind=_kind(oracle, x), plant=plant)
    p = torch.softmax(torch.from_numpy(zt).double() / float(np.float32(T)), -1).numpy()
    return r, p, q


def _position_stats(r, p, q, k=3):
    out = []
    for i in range(k + 1):
        reached = r["accepted_len"] >= i
        tok = r["out_tokens"][reached, i]
        counts = np.bincount(tok, minlength=p.shape[1])
        pval = scipy.stats.chisquare(counts, p[i] * reached.sum()).pvalue
        acc = None
        if i < k:
            n = reached.sum()
            a = (r["accepted_len"][reached] > i).mean()
            alpha = np.minimum(p[i], q[i]).sum()
            acc = (a, alpha, math.sqrt(alpha * (1 - alpha) / n))
        out.append((pval, acc))
    return out


@pytest.mark.parametrize("draft_kind,T,seed", [("probs", 1.0, 0), ("logits", 0.7, 1)])
def test_losslessness_and_acceptance_rate(oracle, draft_kind, T, seed):
    r, p, q = _chain_mc(oracle, draft_kind, T, seed)
    for i, (pval, acc) in enumerate(_position_stats(r, p, q)):
        assert pval > 1e-3, f"position {i}: emitted tokens are not distributed as p (p={pval})"
        if acc is not None:
            a, alpha, sd = acc
            assert abs(a - alpha) < 4 * sd + 1e-12, (i, a, alpha, sd)


@pytest.mark.parametrize("plant", [1, 2])
def test_planted_mistakes_are_caught(oracle, plant):
    """A flipped residual sign (plant 1) or an inverted ratio (plant 2),
    compiled into a copy of the oracle, must fail the losslessness pin."""
    oracle.build(plant=plant)
    r, p, q = _chain_mc(oracle, "probs", 1.0, 0, plant=plant)
    stats = _position_stats(r, p, q)
    assert min(s[0] for s in stats) < 1e-6


# --------------------------------------------------------------------------
# Greedy verification: brute force.
# --------------------------------------------------------------------------
def _quantised_rows(rng, shape, levels=5):
    return rng.integers(-levels, levels + 1, size=shape).astype(np.float32)


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_greedy_chain_bruteforce(oracle, dtype):
    rng = np.random.default_rng(7)
    B, k, V = 300, 4, 40
    z = _quantised_rows(rng, (B, k + 1, V))
    first_max = z.argmax(-1)  # numpy returns the first maximal index
    x = np.where(rng.random((B, k)) < 0.75, first_max[:, :k], rng.integers(0, V, (B, k)))
    zt = inputs._cast(z, dtype)
    r = oracle.verify_chain(zt, None, torch.from_numpy(x.astype(np.int32)), None, 0.0)
    for b in range(B):
        n = 0
        while n < k and x[b, n] == first_max[b, n]:
            n += 1
        assert r["accepted_len"][b] == n
        assert list(r["out_tokens"][b, :n]) == list(x[b, :n])
        assert r["out_tokens"][b, n] == first_max[b, n]
        assert (r["out_tokens"][b, n + 1:] == -1).all()


def _enumerate_tree(z, tok, par):
    """Brute force over all root-to-node paths."""
    n = len(par)
    g = z.argmax(-1)
    best, best_path = 0, [0]
    for j in range(n):
        path = [j]
        while path[-1] != 0:
            path.append(int(par[path[-1]]))
        path = path[::-1]
        ok = all(tok[path[d + 1]] == g[path[d]] for d in range(len(path) - 1))
        if ok and (len(path) > len(best_path)):
            best, best_path = j, path
    return best, best_path, g


def test_tree_greedy_bruteforce(oracle):
    rng = np.random.default_rng(11)
    B, n, V, s = 40, 24, 30, 6
    z = _quantised_rows(rng, (B, n, V), levels=3)
    par = np.full((B, n), -1, np.int32)
    depth = np.zeros((B, n), np.int32)
    tok = np.zeros((B, n), np.int32)
    for b in range(B):
        for j in range(1, n):
            while True:
                pj = int(rng.integers(0, j))
                if depth[b, pj] < s:
                    break
            par[b, j] = pj
            depth[b, j] = depth[b, pj] + 1
            g = int(z[b, pj].argmax())
            tok[b, j] = g if rng.random() < 0.6 else int(rng.integers(0, V))
    r = oracle.tree_greedy(torch.from_numpy(z), torch.from_numpy(tok), torch.from_numpy(par), s)
    for b in range(B):
        best, path, g = _enumerate_tree(z[b], tok[b], par[b])
        L = len(path) - 1
        assert r["accepted_len"][b] == L
        assert list(r["accepted_nodes"][b, :L + 1]) == path
        assert list(r["out_tokens"][b, :L]) == [int(tok[b, j]) for j in path[1:]]
        assert r["out_tokens"][b, L] == g[best]
        assert (r["out_tokens"][b, L + 1:] == -1).all()


def test_chain_shaped_tree_equals_greedy_chain(oracle):
    x = inputs.make_chain(12, 5, 2000, dtype="bf16", sigma_d=0.5, temperature=0.0, seed=4)
    B, P, V = x.target.shape
    par = np.tile(np.arange(-1, P - 1, dtype=np.int32), (B, 1))
    tok = np.concatenate([np.zeros((B, 1), np.int32), x.draft_tokens.numpy()], axis=1)
    t = oracle.tree_greedy(x.target, torch.from_numpy(tok), torch.from_numpy(par), P - 1)
    c = oracle.verify_chain(x.target, None, x.draft_tokens, None, 0.0)
    assert (t["accepted_len"] == c["accepted_len"]).all()
    assert (t["out_tokens"] == c["out_tokens"]).all()
    assert (c["accepted_len"] > 0).any()


# --------------------------------------------------------------------------
# Top-K: a full stable sort (numpy lexsort) and scipy's logsumexp.
# --------------------------------------------------------------------------
@pytest.mark.parametrize("K,T", [(1, 1.0), (7, 0.7), (32, 1.0)])
def test_topk_matches_full_sort(oracle, K, T):
    rng = np.random.default_rng(K)
    z = _quantised_rows(rng, (9, 500), levels=20) / 4
    zt = inputs._cast(z, "bf16")
    zz = zt.double().numpy()
    r = oracle.topk(zt, K, T)
    Tf = float(np.float32(T))
    for row in range(z.shape[0]):
        order = np.lexsort((np.arange(z.shape[1]), -zz[row]))[:K]
        assert list(r["topk_idx"][row]) == list(order)
        lse = scipy.special.logsumexp(zz[row] / Tf)
        assert np.allclose(r["lse"][row], lse, rtol=1e-13)
        assert np.allclose(r["topk_logp"][row], zz[row, order] / Tf - lse, rtol=1e-12, atol=1e-13)


# --------------------------------------------------------------------------
# KL(p~ || q): Gibbs' inequality, the zero case, scipy's rel_entr, V=2.
# --------------------------------------------------------------------------
def test_kl_nonnegative_and_matches_rel_entr(oracle):
    x = inputs.make_chain(6, 3, 4000, dtype="bf16", sigma_d=1.0, temperature=1.0, seed=8)
    tk = oracle.topk(x.target, 32, 1.0)
    d = oracle.kl(tk["topk_logp"], tk["topk_idx"], x.draft, 1.0)
    assert (d["kl"] >= -1e-12).all() and (d["kl"] > 0).all()
    q = torch.softmax(x.draft.double(), -1).numpy()
    for b in range(6):
        for i in range(3):
            pt = scipy.special.softmax(tk["topk_logp"][b, i])
            ref = scipy.special.rel_entr(pt, q[b, i, tk["topk_idx"][b, i]]).sum()
            assert np.isclose(d["kl"][b, i], ref, rtol=1e-11, atol=1e-14)


def test_kl_zero_when_draft_is_renormalised_topk(oracle):
    """q equal to the renormalised top-K of p (draft logits = target logits on
    the kept set, -inf elsewhere) gives KL = 0."""
    x = inputs.make_chain(3, 2, 1000, dtype="f32", sigma_d=0.0, temperature=0.9, seed=9)
    tk = oracle.topk(x.target, 32, 0.9)
    dr = torch.full_like(x.draft, -float("inf"))
    for b in range(3):
        for i in range(2):
            ix = torch.from_numpy(tk["topk_idx"][b, i]).long()
            dr[b, i, ix] = x.target[b, i, ix]
    d = oracle.kl(tk["topk_logp"], tk["topk_idx"], dr, 0.9)
    assert np.abs(d["kl"]).max() < 1e-13


def test_kl_two_token_closed_form(oracle):
    a_t, a_d, T = 0.8, -0.3, 1.0
    zt = torch.tensor([[[a_t, 0.0], [0.0, 0.0]]], dtype=torch.float32)
    zd = torch.tensor([[[a_d, 0.0]]], dtype=torch.float32)
    tk = oracle.topk(zt, 2, T)
    d = oracle.kl(tk["topk_logp"], tk["topk_idx"], zd, T)
    p1 = 1 / (1 + math.exp(-float(np.float32(a_t))))
    q1 = 1 / (1 + math.exp(-float(np.float32(a_d))))
    ref = p1 * math.log(p1 / q1) + (1 - p1) * math.log((1 - p1) / (1 - q1))
    assert math.isclose(d["kl"][0, 0], ref, rel_tol=1e-13)


def test_kl_infinite_when_draft_misses_a_kept_token(oracle):
    zt = torch.tensor([[[1.0, 0.5, 0.0], [0.0, 0.0, 0.0]]])
    q = torch.tensor([[[0.0, 0.5, 0.5]]])
    tk = oracle.topk(zt, 2, 1.0)
    d = oracle.kl(tk["topk_logp"], tk["topk_idx"], q, 1.0, draft_kind=oracle.DRAFT_PROBS)
    assert math.isinf(d["kl"][0, 0]) and d["kl"][0, 0] > 0


# --------------------------------------------------------------------------
# Reward weighting: the pages' worked examples.
# --------------------------------------------------------------------------
def test_kd_loss_worked_example(oracle):
    g = json.load(open(os.path.join(GOLDEN, "respec_kd_loss_example.json")))
    r = oracle.reward_loss(np.array([g["kl"]]), np.array([g["accepted_len"]]),
                           np.array([g["reward"]]), mode=oracle.W_RAW)
    assert math.isclose(r["loss"][0], g["loss"], rel_tol=1e-12)
    assert math.isclose(r["total"], g["loss"], rel_tol=1e-12)
    # Only accepted positions count: two accepted positions drop the third term.
    r2 = oracle.reward_loss(np.array([g["kl"]]), np.array([2]), np.array([g["reward"]]))
    assert math.isclose(r2["loss"][0], g["reward"] * (g["kl"][0] + g["kl"][1]), rel_tol=1e-12)


def test_group_weights_worked_example(oracle):
    g = json.load(open(os.path.join(GOLDEN, "respec_group_weights_example.json")))
    rw = np.array(g["reward"])
    B = len(rw)
    kl = np.full((B, 1), g["kl_each"])
    r = oracle.reward_loss(kl, np.ones(B, np.int32), rw, mode=oracle.W_GROUP_NORM, group=B)
    printed = g["printed_weights"]
    assert np.allclose(np.round(r["w"][:2], g["printed_decimals"]), printed)
    assert r["w"][-1] == g["zero_reward_weight"] and r["loss"][-1] == 0.0
    assert math.isclose(r["w"].sum(), 1.0, rel_tol=1e-12)
    assert np.allclose(r["loss"], r["w"] * g["kl_each"], rtol=1e-12)


def test_group_norm_zero_group_and_clip(oracle):
    rw = np.array([0.0, 0.0, 0.5, 1.5])
    kl = np.ones((4, 2))
    acc = np.array([2, 1, 2, 0], np.int32)
    r = oracle.reward_loss(kl, acc, rw, mode=oracle.W_GROUP_NORM, group=2)
    assert (r["w"][:2] == 0).all() and math.isclose(r["w"][2], 0.25)
    assert r["loss"][3] == 0.0
    rc = oracle.reward_loss(kl, acc, np.array([0.1, 0.7, -2.0, 3.0]), mode=oracle.W_RAW, clip=0.5)
    assert np.allclose(rc["w"], [0.1, 0.5, -0.5, 0.5])


def test_oracle_is_thread_count_invariant(oracle):
    x = inputs.make_chain(24, 3, 3000, dtype="bf16", temperature=0.7, seed=12)
    a = oracle.verify_chain(x.target, x.draft, x.draft_tokens, x.uniforms, 0.7, threads=1)
    b = oracle.verify_chain(x.target, x.draft, x.draft_tokens, x.uniforms, 0.7, threads=8)
    for key in ("accepted_len", "out_tokens", "p_x", "cdf_margin"):
        assert np.array_equal(a[key], b[key], equal_nan=True)
    klen = np.arange(24, dtype=np.int32) % 4
    act = (np.arange(24) % 5 != 0).astype(np.int32)
    a = oracle.verify_chain(x.target, x.draft, x.draft_tokens, x.uniforms, 0.7, threads=1,
                            draft_len=klen, active=act)
    b = oracle.verify_chain(x.target, x.draft, x.draft_tokens, x.uniforms, 0.7, threads=8,
                            draft_len=klen, active=act)
    for key in ("accepted_len", "out_tokens", "cdf_margin"):
        assert np.array_equal(a[key], b[key], equal_nan=True)
    t = inputs.make_tree_sample(B=24, V=500, depth_counts=(3, 3, 2), branching=3, seed=13)
    a = oracle.tree_sample(t.target, t.draft, t.node_tokens, t.parents, t.uniforms,
                           t.temperature, t.max_depth, threads=1)
    b = oracle.tree_sample(t.target, t.draft, t.node_tokens, t.parents, t.uniforms,
                           t.temperature, t.max_depth, threads=8)
    for key in ("accepted_len", "out_tokens", "accepted_nodes", "test_margin", "cdf_margin"):
        assert np.array_equal(a[key], b[key])


# --------------------------------------------------------------------------
# KD gradient into the draft logits (reading notes section 4, Algorithm 1
# step 3: gradient only into the current q_theta; section 5: reward weights).
# --------------------------------------------------------------------------
def _kd_case(seed, B=4, k=2, V=12, K=4, T=0.8):
    rng = np.random.default_rng(seed)
    # logits on a 1/1024 grid: z +- 1/1024 is exact in float32
    draft = np.round(rng.normal(0, 1.5, (B, k, V)) * 1024) / 1024
    lp = np.sort(rng.normal(-2, 1, (B, k + 1, K)), axis=-1)[..., ::-1].copy()
    ix = np.stack([rng.permutation(V)[:K] for _ in range(B * (k + 1))]).reshape(B, k + 1, K)
    acc = np.array([k, 1, 0, 2][:B], np.int32)
    reward = np.array([0.85, 0.3, 0.6, 0.0][:B])
    return draft.astype(np.float32), lp, ix.astype(np.int32), acc, reward, T


def _kd_loss(oracle, draft, lp, ix, acc, reward, T, mode, group, positions=0):
    kl = oracle.kl(lp, ix, torch.from_numpy(draft), T)["kl"]
    return oracle.reward_loss(kl, acc, reward, mode=mode, group=group,
                              positions=positions)["total"]


@pytest.mark.parametrize("mode,group,positions", [(0, 1, 0), (1, 2, 0), (0, 1, 1)])
def test_kd_gradient_matches_central_differences(oracle, mode, group, positions):
    draft, lp, ix, acc, reward, T = _kd_case(3)
    g = oracle.kd_grad(lp, ix, torch.from_numpy(draft), acc, reward, T, mode=mode, group=group,
                       positions=positions)
    h = 1.0 / 1024
    num = np.zeros_like(g)
    for b in range(draft.shape[0]):
        for i in range(draft.shape[1]):
            for j in range(draft.shape[2]):
                zp, zm = draft.copy(), draft.copy()
                zp[b, i, j] += h
                zm[b, i, j] -= h
                num[b, i, j] = (_kd_loss(oracle, zp, lp, ix, acc, reward, T, mode, group,
                                         positions) -
                                _kd_loss(oracle, zm, lp, ix, acc, reward, T, mode, group,
                                         positions)) / (2 * h)
    scale = np.abs(g).max()
    assert scale > 0
    assert np.abs(num - g).max() <= 2e-5 * scale, np.abs(num - g).max() / scale


def test_kd_gradient_rows_sum_to_zero_and_vanish_where_unused(oracle):
    draft, lp, ix, acc, reward, T = _kd_case(4)
    g = oracle.kd_grad(lp, ix, torch.from_numpy(draft), acc, reward, T)
    for b in range(draft.shape[0]):
        for i in range(draft.shape[1]):
            if i >= acc[b] or reward[b] == 0.0:
                assert not g[b, i].any()
            else:
                assert abs(g[b, i].sum()) < 1e-12 * max(1.0, np.abs(g[b, i]).max())
                assert g[b, i].max() > 0 > g[b, i].min()


def test_kd_mask_with_the_first_rejected_position(oracle):
    """positions=1 (the Draft-OPD variant) adds position n when a draft was
    rejected (n < k) and changes nothing when every draft was accepted."""
    rng = np.random.default_rng(5)
    B, k = 6, 3
    kl = rng.uniform(0, 1, (B, k))
    acc = np.array([0, 1, 2, 3, 1, 3], np.int32)
    rw = rng.uniform(0.1, 1, B)
    r0 = oracle.reward_loss(kl, acc, rw)
    r1 = oracle.reward_loss(kl, acc, rw, positions=1)
    for b in range(B):
        n = acc[b]
        extra = rw[b] * kl[b, n] if n < k else 0.0
        assert r1["loss"][b] == pytest.approx(r0["loss"][b] + extra, rel=1e-14, abs=1e-15)
    bumped = np.minimum(acc + 1, k).astype(np.int32)
    r2 = oracle.reward_loss(kl, bumped, rw)
    assert np.allclose(r1["loss"], r2["loss"], rtol=1e-14, atol=0)


# --------------------------------------------------------------------------
# Ragged batches: request b drafted k_b <= k tokens; inactive requests emit
# nothing.
# --------------------------------------------------------------------------
def _ragged_mc(oracle, plant=0):
    rng = np.random.default_rng(31)
    k, V, B = 3, 8, 200_000
    zt = rng.normal(0, 1.5, (k + 1, V)).astype(np.float32)
    d = rng.dirichlet(np.full(V, 0.7), size=k).astype(np.float32)
    x = inputs.make_chain_fixed(B, zt, d, draft_kind="probs", temperature=1.0, seed=9)
    klen = rng.integers(0, k + 1, B).astype(np.int32)
    act = (rng.random(B) < 0.9).astype(np.int32)
    r = oracle.verify_chain(x.target, x.draft, x.draft_tokens, x.uniforms, 1.0,
                            draft_kind=oracle.DRAFT_PROBS, draft_len=klen, active=act,
                            plant=plant)
    p = torch.softmax(torch.from_numpy(zt).double(), -1).numpy()
    return r, p, d.astype(np.float64), klen, act


def _ragged_pvalues(r, p, klen, act):
    k, V = p.shape[0] - 1, p.shape[1]
    acc, out = r["accepted_len"], r["out_tokens"]
    pv = []
    for i in range(k + 1):
        reached = (act == 1) & (klen >= i) & (acc >= i)
        counts = np.bincount(out[reached, i], minlength=V)
        pv.append(scipy.stats.chisquare(counts, p[i] * reached.sum()).pvalue)
    return pv


def test_ragged_planted_bonus_row_is_caught(oracle):
    """A bonus drawn from row k instead of row k_b (plant 3) fails the
    ragged losslessness pin."""
    oracle.build(plant=3)
    r, p, q, klen, act = _ragged_mc(oracle, plant=3)
    assert min(_ragged_pvalues(r, p, klen, act)) < 1e-6


def test_ragged_chain_is_lossless(oracle):
    """With per-request draft lengths k_b the emitted token at every position
    i <= k_b is still distributed as the target row i, and position i < k_b
    accepts at the rate sum_x min(p_i, q_i) (Leviathan et al.); inactive
    requests emit nothing.  A bonus drawn from the wrong row (k instead of
    k_b) fails the chi-square test at position k_b."""
    r, p, q, klen, act = _ragged_mc(oracle)
    k, V = 3, 8
    acc, out = r["accepted_len"], r["out_tokens"]
    off = act == 0
    assert (acc[off] == 0).all() and (out[off] == -1).all()
    on = act == 1
    assert (acc[on] <= klen[on]).all()
    for b in np.flatnonzero(on)[:2000]:
        n = acc[b]
        assert (out[b, n + 1:] == -1).all() and out[b, n] >= 0
    for i, pval in enumerate(_ragged_pvalues(r, p, klen, act)):
        assert pval > 1e-3, (i, pval)
    for i in range(k):
        tested = on & (klen > i) & (acc >= i)
        if tested.any():
            a = (acc[tested] > i).mean()
            alpha = np.minimum(p[i], q[i]).sum()
            sd = math.sqrt(alpha * (1 - alpha) / tested.sum())
            assert abs(a - alpha) < 4 * sd, (i, a, alpha)


def test_ragged_chain_equals_the_shorter_chain(oracle):
    """Request b of a ragged batch gives exactly the result of a chain of
    k_b drafts on the same rows, with the uniforms u_0..u_{k_b} (the draw
    takes u_{k_b}); k_b = 0 is an inverse-CDF draw from the target row 0."""
    T = 0.8
    x = inputs.make_chain(12, 4, 500, dtype="bf16", temperature=T, seed=21)
    klen = np.array([4, 3, 2, 1, 0, 4, 2, 0, 1, 3, 3, 4], np.int32)
    r = oracle.verify_chain(x.target, x.draft, x.draft_tokens, x.uniforms, T, draft_len=klen)
    for b in range(12):
        kb = int(klen[b])
        if kb == 0:
            z = x.target[b, 0].double().numpy() / float(np.float32(T))
            pz = np.exp(z - scipy.special.logsumexp(z))
            u0 = float(x.uniforms[b, 0])
            want = int(np.searchsorted(np.cumsum(pz), u0 * pz.sum(), side="right"))
            assert r["accepted_len"][b] == 0 and r["out_tokens"][b, 0] == want
            assert (r["out_tokens"][b, 1:] == -1).all()
            continue
        s = oracle.verify_chain(x.target[b:b + 1, :kb + 1].contiguous(),
                                x.draft[b:b + 1, :kb].contiguous(),
                                x.draft_tokens[b:b + 1, :kb].contiguous(),
                                x.uniforms[b:b + 1, :kb + 1].contiguous(), T)
        assert r["accepted_len"][b] == s["accepted_len"][0]
        assert list(r["out_tokens"][b, :kb + 1]) == list(s["out_tokens"][0])
        assert (r["out_tokens"][b, kb + 1:] == -1).all()


def test_ragged_greedy_chain_bruteforce(oracle):
    rng = np.random.default_rng(8)
    B, k, V = 200, 4, 30
    z = _quantised_rows(rng, (B, k + 1, V))
    first_max = z.argmax(-1)
    x = np.where(rng.random((B, k)) < 0.8, first_max[:, :k], rng.integers(0, V, (B, k)))
    klen = rng.integers(0, k + 1, B).astype(np.int32)
    act = (rng.random(B) < 0.85).astype(np.int32)
    x[np.arange(k)[None, :] >= klen[:, None]] = -7  # never read: outside the drafts
    x[act == 0] = -7
    r = oracle.verify_chain(torch.from_numpy(z), None, torch.from_numpy(x.astype(np.int32)),
                            None, 0.0, draft_len=klen, active=act)
    for b in range(B):
        if not act[b]:
            assert r["accepted_len"][b] == 0 and (r["out_tokens"][b] == -1).all()
            continue
        n = 0
        while n < klen[b] and x[b, n] == first_max[b, n]:
            n += 1
        assert r["accepted_len"][b] == n
        assert list(r["out_tokens"][b, :n]) == list(x[b, :n])
        assert r["out_tokens"][b, n] == first_max[b, n]
        assert (r["out_tokens"][b, n + 1:] == -1).all()


def test_ragged_kd_mask_and_inactive_requests(oracle):
    """With draft lengths the first-rejected-position rule tests n < k_b, and
    an inactive request contributes nothing to the loss."""
    rng = np.random.default_rng(6)
    B, k = 6, 4
    kl = rng.uniform(0, 1, (B, k))
    klen = np.array([4, 2, 2, 0, 3, 1], np.int32)
    acc = np.array([1, 2, 1, 0, 3, 1], np.int32)
    act = np.array([1, 1, 1, 1, 1, 0], np.int32)
    rw = rng.uniform(0.1, 1, B)
    r = oracle.reward_loss(kl, acc, rw, positions=1, draft_len=klen, active=act)
    want = [rw[0] * kl[0, :2].sum(), rw[1] * kl[1, :2].sum(), rw[2] * kl[2, :2].sum(), 0.0,
            rw[4] * kl[4, :3].sum(), 0.0]
    assert np.allclose(r["loss"], want, rtol=1e-14, atol=0)
    with pytest.raises(oracle.OracleError):
        oracle.reward_loss(kl, np.array([3, 0, 0, 0, 0, 0], np.int32), rw, draft_len=klen * 0 + 2)


# --------------------------------------------------------------------------
# Sampling tree verification (multi-step speculative sampling, SpecInfer).
# --------------------------------------------------------------------------
@pytest.mark.parametrize("draft_kind", ["logits", "probs"])
def test_tree_sample_single_path_equals_chain(oracle, draft_kind):
    """A tree that is one path of k children is chain verification: the same
    ratio tests, the residual at the first rejection, the bonus at the leaf
    (node j+1 tests with the chain's u_j, the final draw takes u_k)."""
    B, k, V, T = 60, 4, 300, 0.8
    x = inputs.make_chain(B, k, V, dtype="bf16", temperature=T, sigma_d=0.6, seed=17)
    draft = x.draft
    kind = oracle.DRAFT_LOGITS
    if draft_kind == "probs":
        draft = torch.softmax(x.draft.float() / float(np.float32(T)), -1)
        kind = oracle.DRAFT_PROBS
    chain = oracle.verify_chain(x.target, draft, x.draft_tokens, x.uniforms, T, draft_kind=kind)
    n = k + 1
    par = np.tile(np.arange(-1, k, dtype=np.int32), (B, 1))
    tok = np.zeros((B, n), np.int32)
    tok[:, 1:] = x.draft_tokens.numpy()
    leaf = draft[:, k - 1:k]  # the leaf's draft row is never used for a test
    tdraft = torch.cat([draft, leaf], dim=1).contiguous()
    u = np.zeros((B, n), np.float32)
    u[:, 1:] = x.uniforms.numpy()[:, :k]
    u[:, 0] = x.uniforms.numpy()[:, k]
    tr = oracle.tree_sample(x.target, tdraft, tok, par, u, T, k, draft_kind=kind)
    assert np.array_equal(tr["accepted_len"], chain["accepted_len"])
    assert np.array_equal(tr["out_tokens"], chain["out_tokens"])
    for b in range(B):
        a = tr["accepted_len"][b]
        assert list(tr["accepted_nodes"][b, :a + 1]) == list(range(a + 1))
    assert len(set(chain["accepted_len"].tolist())) > 2


def _tree_mc(oracle, plant=0, B=200_000, V=5, m1=3, m2=2, seed=23):
    """Depth-2 trees whose rows depend only on the path's tokens: the root's
    m1 children and each depth-1 node's m2 children are drawn independently
    from the draft row of their parent's context."""
    rng = np.random.default_rng(seed)
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
    tok[:, 1:1 + m1] = rng.choice(V, size=(B, m1), p=q0)
    cum1 = np.cumsum(q1, axis=1)
    for i in range(m1):
        t1 = tok[:, 1 + i]
        draws = (rng.random((B, m2))[:, :, None] > cum1[t1][:, None, :]).sum(-1)
        tok[:, 1 + m1 + i * m2:1 + m1 + (i + 1) * m2] = np.minimum(draws, V - 1)
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
            qd[:, c] = q0  # a leaf's draft row is never used for a test
    u = inputs.uniforms24(np.random.default_rng(seed + 1), (B, n))
    r = oracle.tree_sample(torch.from_numpy(logp), torch.from_numpy(qd), tok, par, u, 1.0, 2,
                           draft_kind=oracle.DRAFT_PROBS, plant=plant)
    # the target rows as stored (fp32 log-probabilities, renormalised at T = 1)
    def sm(z):
        z = z.astype(np.float64)
        e = np.exp(z - z.max(-1, keepdims=True))
        return e / e.sum(-1, keepdims=True)
    return r, sm(np.log(p0).astype(np.float32)), sm(np.log(p1).astype(np.float32)), \
        sm(np.log(p2).astype(np.float32)), q0.astype(np.float32).astype(np.float64)


def _tree_pvalues(r, P0, P1, P2, min_count=400):
    acc, out = r["accepted_len"], r["out_tokens"]
    V = P0.shape[0]
    pv = [scipy.stats.chisquare(np.bincount(out[:, 0], minlength=V), P0 * len(acc)).pvalue]
    for t in range(V):
        sel = (acc >= 1) & (out[:, 0] == t)
        if sel.sum() >= min_count:
            pv.append(scipy.stats.chisquare(np.bincount(out[sel, 1], minlength=V),
                                            P1[t] * sel.sum()).pvalue)
        for t2 in range(V):
            sel2 = sel & (acc >= 2) & (out[:, 1] == t2)
            if sel2.sum() >= min_count:
                pv.append(scipy.stats.chisquare(np.bincount(out[sel2, 2], minlength=V),
                                                P2[t, t2] * sel2.sum()).pvalue)
    return pv


def test_tree_sample_is_lossless(oracle):
    """Every emitted token follows the target row of its context (SpecInfer's
    theorem for multi-step speculative sampling), at all three positions; the
    root rejects all m children with probability prod_i (1 - sum_x min(q, r_i)),
    r_0 = p and r_{i+1} the normalised max(0, r_i - q)."""
    r, P0, P1, P2, q0 = _tree_mc(oracle)
    pv = _tree_pvalues(r, P0, P1, P2)
    assert len(pv) > 10
    assert min(pv) > 1e-4, pv
    rr, none = P0.copy(), 1.0
    for _ in range(3):
        none *= 1.0 - np.minimum(q0, rr).sum()
        rr = np.maximum(rr - q0, 0.0)
        rr /= rr.sum()
    got = (r["accepted_len"] == 0).mean()
    sd = math.sqrt(none * (1 - none) / len(r["accepted_len"]))
    assert abs(got - none) < 4 * sd, (got, none)
    assert (r["fallback"] == 0).all()


def test_tree_sample_planted_sibling_mistake_is_caught(oracle):
    """Testing every sibling against p instead of the running residual (plant
    4) over-accepts drafted tokens and must fail the losslessness pin."""
    oracle.build(plant=4)
    r, P0, P1, P2, _ = _tree_mc(oracle, plant=4)
    assert min(_tree_pvalues(r, P0, P1, P2)) < 1e-6


def test_tree_sample_rejects_malformed_trees(oracle):
    z = torch.zeros(1, 3, 4)
    tok = np.array([[0, 1, 2]], np.int32)
    u = np.full((1, 3), 0.5, np.float32)
    for par, depth in (([[-1, 0, 2]], 2), ([[0, 0, 1]], 2), ([[-1, 0, 1]], 1)):
        with pytest.raises(oracle.OracleError):
            oracle.tree_sample(z, z, tok, np.array(par, np.int32), u, 1.0, depth)
