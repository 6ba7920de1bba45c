"""Parity of the CUDA path (through the C ABI) with the float64 oracle, on the
workloads (tiny fp32 chain; Qwen-vocabulary chain; the active-batch sweep;
greedy trees; fused verify + KD) and on edge cases.  See tests/parity.py for
the comparison rules."""
import numpy as np
import pytest
import torch

from oracle import oracle as O
from speculative_decoding_verification_94_b200 import inputs, sv
from tests.parity import assert_chain_match, assert_close, assert_kd_match, bitwise_equal

pytestmark = pytest.mark.gpu

DEV = "cuda"


def status_tensor():
    return torch.zeros(1, dtype=torch.int32, device=DEV)


def run_chain(x, kd=None, status=None, **kw):
    return sv.sv_verify_chain(x.target.to(DEV), x.draft.to(DEV) if x.draft is not None else None,
                              x.draft_tokens.to(DEV),
                              x.uniforms.to(DEV) if x.uniforms is not None else None,
                              x.temperature, draft_kind=x.draft_kind, kd=kd,
                              device_status=status, **kw)


def oracle_chain(x):
    kind = O.DRAFT_PROBS if x.draft_kind == "probs" else O.DRAFT_LOGITS
    return O.verify_chain(x.target, x.draft, x.draft_tokens, x.uniforms, x.temperature,
                          draft_kind=kind)


def check_chain(x, max_flag_frac=0.05):
    st = status_tensor()
    got = run_chain(x, status=st)
    torch.cuda.synchronize()
    assert int(st.item()) & sv.SV_DEV_ERROR_MASK == 0
    ref = oracle_chain(x)
    return assert_chain_match(got, ref, x.uniforms.numpy(), x.temperature, x.k, max_flag_frac)


CHAIN_PATHS = {"two-kernel": {}, "two-kernel-direct": dict(finish_read=2),
               "persistent": dict(persistent=1)}


@pytest.fixture(params=list(CHAIN_PATHS))
def chain_path(request):
    """Run the test on every chain path: the default two-kernel path (its
    finishing clusters staging the drawn row in shared memory, or reading it
    from global memory) and the single persistent launch."""
    with sv.knobs(**CHAIN_PATHS[request.param]):
        yield request.param


# --------------------------------------------------------------------------
# Workloads
# --------------------------------------------------------------------------
def test_tiny_chain_fp32(chain_path):
    r = check_chain(inputs.tiny_chain(seed=0))
    assert r["flagged"] == 0


@pytest.fixture(scope="module")
def qwen32():
    return inputs.qwen_chain(B=32, k=3, sigma_d=1.0, seed=0)


def test_qwen_chain_full_size(qwen32, chain_path):
    r = check_chain(qwen32)
    print("qwen chain", r)


@pytest.mark.parametrize("k", [1, 3, 5, 7])
@pytest.mark.parametrize("sigma", [0.3, 1.0, 3.0])
def test_active_batch_sweep(k, sigma, chain_path):
    x = inputs.qwen_chain(B=32, k=k, sigma_d=sigma, seed=100 + k)
    ref = oracle_chain(x)
    for B in (1, 2, 4, 8, 16, 32):
        sub = inputs.ChainInputs(x.target[:B].contiguous(), x.draft[:B].contiguous(),
                                 x.draft_tokens[:B].contiguous(), x.uniforms[:B].contiguous(),
                                 x.reward[:B], x.temperature)
        got = run_chain(sub)
        torch.cuda.synchronize()
        refb = {key: v[:B] for key, v in ref.items() if isinstance(v, np.ndarray)}
        assert_chain_match(got, refb, sub.uniforms.numpy(), x.temperature, k, max_flag_frac=0.2)


def test_tree_greedy_full_size():
    t = inputs.make_tree(B=8, seed=0)
    st = status_tensor()
    got = sv.sv_verify_tree_greedy(t.logits.to(DEV), t.node_tokens.to(DEV), t.parents.to(DEV),
                                   t.max_depth, device_status=st)
    ref = O.tree_greedy(t.logits, t.node_tokens, t.parents, t.max_depth)
    torch.cuda.synchronize()
    assert int(st.item()) == 0
    for key in ("accepted_len", "out_tokens", "accepted_nodes"):
        assert np.array_equal(got[key].cpu().numpy(), ref[key]), key
    assert len(set(ref["accepted_len"].tolist())) > 1
    # the workspace (stream records, row records, arrival counts) is zero again
    assert int(torch.count_nonzero(sv._WS[torch.cuda.current_device()])) == 0


@pytest.mark.parametrize("n,depth", [(8, 3), (9, 4), (40, 6), (130, 9)])
def test_tree_greedy_node_counts(n, depth):
    """Trees of fewer nodes than a block's warps (one block), just over them
    (two blocks per tree) and of several blocks per tree, against path
    enumeration in the oracle; the workspace is zero afterwards."""
    rng = np.random.default_rng(n)
    B, V = 6, 3001
    par = np.full((B, n), -1, np.int32)
    for b in range(B):
        depth_of = [0]
        for j in range(1, n):
            cand = [i for i in range(j) if depth_of[i] < depth]
            p = int(rng.choice(cand))
            par[b, j] = p
            depth_of.append(depth_of[p] + 1)
    logits = torch.from_numpy(rng.normal(0, 2, (B, n, V)).astype(np.float32))
    am = logits.argmax(-1).numpy()
    tok = rng.integers(0, V, (B, n)).astype(np.int32)
    for b in range(B):  # plant argmax children so that paths of several depths are accepted
        for j in range(1, n):
            if rng.random() < 0.6:
                tok[b, j] = am[b, par[b, j]]
    st = status_tensor()
    got = sv.sv_verify_tree_greedy(logits.to(DEV), torch.from_numpy(tok).to(DEV),
                                   torch.from_numpy(par).to(DEV), depth, device_status=st)
    ref = O.tree_greedy(logits, torch.from_numpy(tok), torch.from_numpy(par), depth)
    torch.cuda.synchronize()
    assert int(st.item()) == 0
    for key in ("accepted_len", "out_tokens", "accepted_nodes"):
        assert np.array_equal(got[key].cpu().numpy(), ref[key]), key
    assert int(torch.count_nonzero(sv._WS[torch.cuda.current_device()])) == 0


@pytest.fixture(scope="module")
def kd256():
    return inputs.kd_chain(B=256, k=3, seed=0)


@pytest.mark.parametrize("wmode,group", [("raw", 1), ("group_norm", 16)])
def test_fused_verify_kd_full_size(kd256, wmode, group, chain_path):
    x = kd256
    st = status_tensor()
    kd = dict(K=32, reward=x.reward.to(DEV), wmode=wmode, group=group, clip=0.0)
    got = run_chain(x, kd=kd, status=st)
    torch.cuda.synchronize()
    assert int(st.item()) & sv.SV_DEV_ERROR_MASK == 0
    ref = O.verify_kd(x.target, x.draft, x.draft_tokens, x.uniforms, x.reward, x.temperature, 32,
                      mode=O.W_GROUP_NORM if wmode == "group_norm" else O.W_RAW, group=group)
    r = assert_chain_match(got, ref, x.uniforms.numpy(), x.temperature, x.k)
    print("kd verify", r)
    assert_kd_match(got, ref, x.k)
    # loss / total against the oracle's KL and the GPU's own accepted lengths
    acc = got["accepted_len"].cpu().numpy()
    rl = O.reward_loss(ref["kl"], acc, x.reward.numpy().astype(np.float64),
                       mode=O.W_GROUP_NORM if wmode == "group_norm" else O.W_RAW, group=group)
    mag = np.array([abs(rl["w"][b]) * ref["scale"][b, :max(acc[b], 0)].sum() for b in range(x.B)])
    assert_close(got["loss"].cpu().numpy(), rl["loss"], mag, "loss")
    assert_close(got["total"].cpu().numpy(), [rl["total"]], [mag.sum()], "total")


def test_topk_standalone(qwen32):
    x = qwen32
    got = sv.sv_extract_topk_kd(x.target.to(DEV), 32, x.temperature)
    ref = O.topk(x.target, 32, x.temperature)
    torch.cuda.synchronize()
    assert np.array_equal(got["topk_idx"].cpu().numpy(), ref["topk_idx"])
    assert_close(got["topk_logp"].cpu().numpy(), ref["topk_logp"], 1.0, "topk_logp")
    assert_close(got["lse"].cpu().numpy(), ref["lse"], 1.0, "lse")


@pytest.mark.parametrize("draft_kind", ["logits", "probs"])
def test_kl_loss_standalone(qwen32, draft_kind):
    x = qwen32
    draft = x.draft
    if draft_kind == "probs":
        draft = torch.softmax(x.draft.float() / x.temperature, dim=-1)
    tk = O.topk(x.target, 32, x.temperature)
    acc = torch.tensor(np.arange(x.B) % (x.k + 1), dtype=torch.int32)
    st = status_tensor()
    got = sv.sv_kd_kl_loss(torch.from_numpy(tk["topk_logp"].astype(np.float32)).to(DEV),
                           torch.from_numpy(tk["topk_idx"]).to(DEV), draft.to(DEV), x.temperature,
                           acc.to(DEV), x.reward.to(DEV), draft_kind=draft_kind,
                           wmode="group_norm", group=8, clip=0.5, device_status=st)
    torch.cuda.synchronize()
    assert int(st.item()) == 0
    ref = O.kl(tk["topk_logp"], tk["topk_idx"], draft, x.temperature,
               draft_kind=O.DRAFT_PROBS if draft_kind == "probs" else O.DRAFT_LOGITS)
    assert_close(got["kl"].cpu().numpy(), ref["kl"], ref["scale"], "kl")
    rl = O.reward_loss(ref["kl"], acc.numpy(), x.reward.numpy().astype(np.float64),
                       mode=O.W_GROUP_NORM, group=8, clip=0.5)
    mag = np.array([abs(rl["w"][b]) * ref["scale"][b, :acc[b]].sum() for b in range(x.B)])
    assert_close(got["loss"].cpu().numpy(), rl["loss"], mag, "loss")
    assert_close(got["total"].cpu().numpy(), [rl["total"]], [mag.sum()], "total")


# --------------------------------------------------------------------------
# Losslessness on the GPU itself (Leviathan): emitted tokens follow p.
# --------------------------------------------------------------------------
def test_gpu_losslessness_chi_square(chain_path):
    import scipy.stats
    rng = np.random.default_rng(5)
    V, k, B = 8, 3, 1_000_000
    zt = rng.normal(0, 1.5, (k + 1, V)).astype(np.float32)
    q = rng.dirichlet(np.full(V, 0.7), size=k).astype(np.float32)
    x = inputs.make_chain_fixed(B, zt, q, draft_kind="probs", temperature=1.0, seed=21)
    got = run_chain(x)
    acc = got["accepted_len"].cpu().numpy()
    out = got["out_tokens"].cpu().numpy()
    p = torch.softmax(torch.from_numpy(zt).double(), -1).numpy()
    for i in range(k + 1):
        reached = acc >= i
        counts = np.bincount(out[reached, i], minlength=V)
        assert scipy.stats.chisquare(counts, p[i] * reached.sum()).pvalue > 1e-3, i
        if i < k:
            alpha = np.minimum(p[i], q[i].astype(np.float64)).sum()
            a = (acc[reached] > i).mean()
            assert abs(a - alpha) < 4 * np.sqrt(alpha * (1 - alpha) / reached.sum())
    # and request by request against the oracle on a slice
    sl = slice(0, 20000)
    sub = inputs.ChainInputs(x.target[sl], x.draft[sl], x.draft_tokens[sl], x.uniforms[sl],
                             x.reward[sl], 1.0, draft_kind="probs")
    ref = oracle_chain(sub)
    assert_chain_match({"accepted_len": torch.from_numpy(acc[sl]),
                        "out_tokens": torch.from_numpy(out[sl])}, ref, sub.uniforms.numpy(), 1.0,
                       k, max_flag_frac=0.001)


# --------------------------------------------------------------------------
# Edge cases
# --------------------------------------------------------------------------
@pytest.mark.parametrize("V", [1, 2, 7, 8, 64, 1001, 4099, 70001, 151936])
@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_ragged_and_small_vocab(V, dtype, chain_path):
    x = inputs.make_chain(12, 3, V, dtype=dtype, model="zipf" if V > 64 else "gauss",
                          sigma_t=2.0, sigma_d=1.0, temperature=0.9, seed=V)
    check_chain(x, max_flag_frac=0.25)


@pytest.mark.parametrize("k", [1, 15, 30, 31, 40])
def test_k_extremes(k, chain_path):
    """k <= 30 runs as one persistent launch, k > 30 on the two-kernel path."""
    check_chain(inputs.make_chain(12, k, 5000, dtype="bf16", sigma_d=0.3, temperature=1.0,
                                  seed=k), max_flag_frac=0.25)


def test_empty_batch(chain_path):
    x = inputs.make_chain(1, 3, 100, dtype="f32", seed=1)
    z = torch.empty(0, 4, 100, device=DEV)
    d = torch.empty(0, 3, 100, device=DEV)
    got = sv.sv_verify_chain(z, d, torch.empty(0, 3, dtype=torch.int32, device=DEV),
                             torch.empty(0, 4, device=DEV), 1.0)
    assert got["accepted_len"].numel() == 0
    del x


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_draft_probabilities(dtype, chain_path):
    x = inputs.make_chain(16, 3, 3000, dtype=dtype, sigma_d=1.0, temperature=0.8, seed=3)
    probs = torch.softmax(x.draft.float() / x.temperature, dim=-1).contiguous()
    y = inputs.ChainInputs(x.target, probs, x.draft_tokens, x.uniforms, x.reward, x.temperature,
                           draft_kind="probs")
    check_chain(y)


def test_identical_draft_accepts_everything_on_gpu(chain_path):
    x = inputs.make_chain(64, 4, 30000, dtype="bf16", sigma_d=0.0, temperature=0.7, seed=9)
    got = run_chain(x)
    assert (got["accepted_len"].cpu() == 4).all()
    check_chain(x)


def test_disjoint_support_on_gpu(chain_path):
    V, k, B = 4096, 3, 128
    rng = np.random.default_rng(0)
    zt = rng.normal(0, 2, (k + 1, V)).astype(np.float32)
    zd = rng.normal(0, 2, (k, V)).astype(np.float32)
    zt[:, 1::2] = -np.inf
    zd[:, 0::2] = -np.inf
    for dtype in ("f32", "bf16"):
        x = inputs.make_chain_fixed(B, zt, zd, draft_kind="logits", temperature=1.0, seed=1,
                                    dtype=dtype)
        got = run_chain(x)
        assert (got["accepted_len"].cpu() == 0).all()
        assert (got["out_tokens"][:, 0].cpu() % 2 == 0).all()
        check_chain(x)


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_greedy_chain_with_ties(dtype, chain_path):
    rng = np.random.default_rng(7)
    B, k, V = 64, 4, 3000
    z = rng.integers(-3, 4, size=(B, k + 1, V)).astype(np.float32)
    first = z.argmax(-1)
    xt = np.where(rng.random((B, k)) < 0.8, first[:, :k], rng.integers(0, V, (B, k)))
    zt = inputs._cast(z, dtype)
    tok = torch.from_numpy(xt.astype(np.int32))
    got = sv.sv_verify_chain(zt.to(DEV), None, tok.to(DEV), None, 0.0)
    ref = O.verify_chain(zt, None, tok, None, 0.0)
    assert np.array_equal(got["accepted_len"].cpu().numpy(), ref["accepted_len"])
    assert np.array_equal(got["out_tokens"].cpu().numpy(), ref["out_tokens"])


def test_greedy_chain_full_size(qwen32, chain_path):
    x = qwen32
    tok = x.target[:, :3].float().argmax(-1).to(torch.int32)
    tok[::3, 1] = 5
    got = sv.sv_verify_chain(x.target.to(DEV), None, tok.to(DEV), None, 0.0)
    ref = O.verify_chain(x.target, None, tok, None, 0.0)
    assert np.array_equal(got["accepted_len"].cpu().numpy(), ref["accepted_len"])
    assert np.array_equal(got["out_tokens"].cpu().numpy(), ref["out_tokens"])


def test_topk_with_massive_ties_and_small_rows():
    z = torch.zeros(3, 50000)
    z[1, 123] = 1.0
    z[2, :10] = torch.arange(10, dtype=torch.float32)
    for dtype in (torch.float32, torch.bfloat16):
        zz = z.to(dtype)
        st = status_tensor()
        got = sv.sv_extract_topk_kd(zz.to(DEV), 32, 1.0, device_status=st)
        ref = O.topk(zz, 32, 1.0)
        torch.cuda.synchronize()
        assert np.array_equal(got["topk_idx"].cpu().numpy(), ref["topk_idx"])
        assert_close(got["topk_logp"].cpu().numpy(), ref["topk_logp"], 1.0, "topk_logp")
        assert int(st.item()) & sv.SV_DEV_ERROR_MASK == 0
    small = torch.randn(7, 40)
    got = sv.sv_extract_topk_kd(small.to(DEV), 32, 0.5)
    ref = O.topk(small, 32, 0.5)
    assert np.array_equal(got["topk_idx"].cpu().numpy(), ref["topk_idx"])
    assert_close(got["topk_logp"].cpu().numpy(), ref["topk_logp"], 1.0, "topk_logp")


def test_device_checks_flag_bad_inputs(chain_path):
    x = inputs.make_chain(4, 3, 500, dtype="f32", seed=2)
    tok = x.draft_tokens.clone()
    tok[1, 0] = 500  # out of range (position 0 is always verified)
    st = status_tensor()
    got = sv.sv_verify_chain(x.target.to(DEV), x.draft.to(DEV), tok.to(DEV), x.uniforms.to(DEV),
                             1.0, device_status=st)
    torch.cuda.synchronize()
    assert int(st.item()) & sv.SV_DEV_BAD_TOKEN
    assert got["accepted_len"][1].item() == -1
    assert (got["out_tokens"][1].cpu() == -1).all()
    # a target row with no finite logit
    t = x.target.clone()
    t[2, 0] = -float("inf")
    st.zero_()
    got = sv.sv_verify_chain(t.to(DEV), x.draft.to(DEV), x.draft_tokens.to(DEV),
                             x.uniforms.to(DEV), 1.0, device_status=st)
    torch.cuda.synchronize()
    assert int(st.item()) & sv.SV_DEV_NO_FINITE
    assert got["accepted_len"][2].item() == -1
    # a malformed tree
    tr = inputs.make_tree(B=2, V=300, seed=1)
    par = tr.parents.clone()
    par[1, 5] = 7  # parent after child
    st.zero_()
    got = sv.sv_verify_tree_greedy(tr.logits.to(DEV), tr.node_tokens.to(DEV), par.to(DEV),
                                   tr.max_depth, device_status=st)
    torch.cuda.synchronize()
    assert int(st.item()) & sv.SV_DEV_BAD_TREE
    assert got["accepted_len"][1].item() == -1
    assert got["accepted_len"][0].item() >= 0


def test_zero_residual_falls_back_to_target(chain_path):
    """p == q but x outside both supports: rejected with zero residual mass."""
    V = 64
    z = np.random.default_rng(1).normal(0, 1, (4, V)).astype(np.float32)
    z[:, 5] = -np.inf
    x = inputs.make_chain_fixed(8, z, z[:3], draft_kind="logits", temperature=1.0, seed=4)
    x.draft_tokens[:] = 5
    st = status_tensor()
    got = run_chain(x, status=st)
    torch.cuda.synchronize()
    assert int(st.item()) & sv.SV_DEV_RESIDUAL_ZERO
    ref = oracle_chain(x)
    assert (ref["fallback"] == 1).all()
    assert_chain_match(got, ref, x.uniforms.numpy(), 1.0, 3)


def test_deterministic_and_workspace_reuse(kd256, chain_path):
    x = kd256
    kd = dict(K=32, reward=x.reward.to(DEV), wmode="group_norm", group=16)
    a = run_chain(x, kd=kd)
    b = run_chain(x, kd=kd)
    torch.cuda.synchronize()
    for key in a:
        assert bitwise_equal(a[key], b[key]), key
    # a smaller batch on the same (cached) workspace, then the full one again
    sub = inputs.ChainInputs(x.target[:16].contiguous(), x.draft[:16].contiguous(),
                             x.draft_tokens[:16].contiguous(), x.uniforms[:16].contiguous(),
                             x.reward[:16].contiguous(), x.temperature)
    s = run_chain(sub, kd=dict(K=32, reward=sub.reward.to(DEV), wmode="group_norm", group=16))
    torch.cuda.synchronize()
    assert torch.equal(s["accepted_len"], a["accepted_len"][:16])
    assert torch.equal(s["out_tokens"], a["out_tokens"][:16])
    assert torch.equal(s["topk_idx"], a["topk_idx"][:16])
    c = run_chain(x, kd=kd)
    torch.cuda.synchronize()
    for key in a:
        assert bitwise_equal(a[key], c[key]), key


@pytest.mark.parametrize("C", [1, 2, 3, 4, 8, 12, 16])
def test_every_cluster_size(C):
    """The two-kernel path's finishing cluster size must not change any result."""
    with sv.knobs(cluster_ctas=C):
        x = inputs.make_chain(24, 3, 20000, dtype="bf16", sigma_d=1.0, temperature=0.7, seed=C)
        check_chain(x, max_flag_frac=0.2)
        got = sv.sv_extract_topk_kd(x.target.to(DEV), 32, 0.7)
        ref = O.topk(x.target, 32, 0.7)
        assert np.array_equal(got["topk_idx"].cpu().numpy(), ref["topk_idx"])


PATHS = {"persistent": dict(persistent=1), "persistent-order1": dict(persistent=1, order=1),
         "persistent-order2-stages2": dict(persistent=1, order=2, stages=2),
         "two-kernel-static": dict(stream_count=1), "two-kernel-dynamic": dict(stream_count=2)}


@pytest.mark.parametrize("path", list(PATHS))
def test_both_stream_schedules(kd256, path):
    """Every chain path gives the oracle's results: the persistent kernel in
    both tile orders and with a shallow ring, and the two-kernel path with its
    static partition (rows completed by the finisher) and its dynamic items
    (in-stream counting and early exit); the workspace is all zero after every
    call."""
    with sv.knobs(**PATHS[path]):
        _schedule_case(kd256)


def _schedule_case(kd256):
    x = kd256
    st = status_tensor()
    kd = dict(K=32, reward=x.reward.to(DEV), wmode="group_norm", group=16)
    got = run_chain(x, kd=kd, status=st)
    torch.cuda.synchronize()
    assert int(st.item()) & sv.SV_DEV_ERROR_MASK == 0
    ref = O.verify_kd(x.target, x.draft, x.draft_tokens, x.uniforms, x.reward, x.temperature, 32,
                      mode=O.W_GROUP_NORM, group=16)
    assert_chain_match(got, ref, x.uniforms.numpy(), x.temperature, x.k)
    assert_kd_match(got, ref, x.k)
    ws = sv._WS[torch.cuda.current_device()]
    assert int(torch.count_nonzero(ws)) == 0
    # plain sampling and greedy chains under the same schedule
    check_chain(inputs.make_chain(48, 3, 70001, dtype="bf16", sigma_d=1.0, temperature=0.7,
                                  seed=7))
    g = inputs.make_chain(48, 3, 70001, dtype="bf16", sigma_d=1.0, temperature=0.0, seed=8)
    got = run_chain(g)
    ref = oracle_chain(g)
    torch.cuda.synchronize()
    assert np.array_equal(got["accepted_len"].cpu().numpy(), ref["accepted_len"])
    assert np.array_equal(got["out_tokens"].cpu().numpy(), ref["out_tokens"])
    assert int(torch.count_nonzero(ws)) == 0


def _grad_check(x, acc, reward, ref_top, mode, group, T, positions=0):
    """sv_kd_grad against the oracle on the same top-K buffers and lengths,
    element by element."""
    lp = torch.from_numpy(ref_top["topk_logp"].astype(np.float32))
    ix = torch.from_numpy(ref_top["topk_idx"].astype(np.int32))
    st = status_tensor()
    got = sv.sv_kd_grad(lp.to(DEV), ix.to(DEV), x.draft.to(DEV),
                        torch.from_numpy(acc).to(DEV), x.reward.to(DEV), T,
                        wmode="group_norm" if mode == O.W_GROUP_NORM else "raw", group=group,
                        positions=positions, device_status=st)
    torch.cuda.synchronize()
    assert int(st.item()) & sv.SV_DEV_ERROR_MASK == 0
    ref = O.kd_grad(lp.numpy().astype(np.float64), ix.numpy(), x.draft, acc,
                    x.reward.numpy().astype(np.float64), T, mode=mode, group=group,
                    positions=positions)
    g = got.cpu().numpy().astype(np.float64)
    # tolerance: 1e-5 of the magnitude the rounding acts on, |w|/T (q_j + p~_j)
    w = O.reward_loss(np.zeros((x.B, x.k)), acc, x.reward.numpy().astype(np.float64),
                      mode=mode, group=group, positions=positions)["w"]
    q = O.softmax(x.draft, T)["p"].reshape(x.B, x.k, -1)
    mag = q.copy()
    B, P, K = lp.shape
    pt = np.exp(lp.numpy() - np.log(np.exp(lp.numpy().astype(np.float64)).sum(-1, keepdims=True)))
    for b in range(B):
        for i in range(x.k):
            mag[b, i, ix[b, i].numpy()] += pt[b, i]
    mag *= (np.abs(w) / T)[:, None, None]
    err = np.abs(g - ref)
    worst = float((err / np.maximum(mag, 1e-300)).max())
    print(f"kd_grad: worst error {worst:.3e} of the element's magnitude (bar 1e-5)")
    assert (err <= 1e-5 * mag + 1e-30).all(), worst
    m = np.where((acc < x.k) & (positions != 0), acc + 1, acc)
    active = np.arange(x.k)[None, :] < m[:, None]
    assert not g[~active].any()
    # the workspace (records and the per-row fold counts of split rows) is zero again
    ws = sv._WS[torch.cuda.current_device()]
    assert int(torch.count_nonzero(ws)) == 0
    return got


def test_kd_grad_small_and_ragged():
    x = inputs.make_chain(6, 3, 1001, dtype="f32", model="gauss", sigma_t=2.0, sigma_d=0.5,
                          temperature=1.0, seed=21)
    ref = O.verify_kd(x.target, x.draft, x.draft_tokens, x.uniforms, x.reward, 1.0, 8)
    acc = ref["accepted_len"].astype(np.int32)
    acc[0] = 3  # at least one request with every draft kept
    _grad_check(x, acc, x.reward, ref, O.W_RAW, 1, 1.0)


def test_kd_grad_split_rows_with_unaligned_tails():
    """V = 8193: each draft row is split over several CTAs (the last one
    ragged), odd rows start off a 16-byte boundary (scalar path) and the
    last vector of a row is partial."""
    x = inputs.make_chain(8, 3, 8193, dtype="bf16", sigma_d=1.0, temperature=0.9, seed=23)
    ref = O.verify_kd(x.target, x.draft, x.draft_tokens, x.uniforms, x.reward, 0.9, 32,
                      mode=O.W_GROUP_NORM, group=4)
    acc = ref["accepted_len"].astype(np.int32)
    acc[0] = 3
    _grad_check(x, acc, x.reward, ref, O.W_GROUP_NORM, 4, 0.9)


def test_kd_grad_full_vocabulary(kd256):
    x = inputs.ChainInputs(kd256.target[:32].contiguous(), kd256.draft[:32].contiguous(),
                           kd256.draft_tokens[:32].contiguous(), kd256.uniforms[:32].contiguous(),
                           kd256.reward[:32].contiguous(), kd256.temperature)
    ref = O.verify_kd(x.target, x.draft, x.draft_tokens, x.uniforms, x.reward, x.temperature, 32,
                      mode=O.W_GROUP_NORM, group=16)
    acc = ref["accepted_len"].astype(np.int32)
    _grad_check(x, acc, x.reward, ref, O.W_GROUP_NORM, 16, x.temperature)


def test_kd_first_rejected_position(kd256, chain_path):
    """positions=1 (the Draft-OPD variant): the loss and the gradient also
    cover the first rejected position."""
    x = inputs.ChainInputs(kd256.target[:32].contiguous(), kd256.draft[:32].contiguous(),
                           kd256.draft_tokens[:32].contiguous(), kd256.uniforms[:32].contiguous(),
                           kd256.reward[:32].contiguous(), kd256.temperature)
    st = status_tensor()
    kd = dict(K=32, reward=x.reward.to(DEV), wmode="group_norm", group=16, positions=1)
    got = run_chain(x, kd=kd, status=st)
    torch.cuda.synchronize()
    assert int(st.item()) & sv.SV_DEV_ERROR_MASK == 0
    ref = O.verify_kd(x.target, x.draft, x.draft_tokens, x.uniforms, x.reward, x.temperature, 32,
                      mode=O.W_GROUP_NORM, group=16, positions=1)
    assert_chain_match(got, ref, x.uniforms.numpy(), x.temperature, x.k)
    acc = got["accepted_len"].cpu().numpy()
    assert (acc < x.k).any()
    rl = O.reward_loss(ref["kl"], acc, x.reward.numpy().astype(np.float64), mode=O.W_GROUP_NORM,
                       group=16, positions=1)
    m = np.where(acc < x.k, acc + 1, acc)
    mag = np.array([abs(rl["w"][b]) * ref["scale"][b, :m[b]].sum() for b in range(x.B)])
    assert_close(got["loss"].cpu().numpy(), rl["loss"], mag, "loss")
    assert_close(got["total"].cpu().numpy(), [rl["total"]], [mag.sum()], "total")
    # the standalone loss and the gradient with the same positions
    lp = torch.from_numpy(ref["topk_logp"].astype(np.float32))
    ix = torch.from_numpy(ref["topk_idx"].astype(np.int32))
    accd = torch.from_numpy(acc.astype(np.int32)).to(DEV)
    kl = sv.sv_kd_kl_loss(lp.to(DEV), ix.to(DEV), x.draft.to(DEV), x.temperature, accd,
                          x.reward.to(DEV), wmode="group_norm", group=16, positions=1)
    torch.cuda.synchronize()
    assert_close(kl["loss"].cpu().numpy(), rl["loss"], mag, "standalone loss")
    # the gradient with the same positions, element by element at 1e-5
    _grad_check(x, acc.astype(np.int32), x.reward, ref, O.W_GROUP_NORM, 16, x.temperature,
                positions=1)
