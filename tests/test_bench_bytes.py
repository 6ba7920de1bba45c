"""The benchmark's byte counts (the numerators of its roofline figures),
checked on CPU against sums written out from the tensors themselves: the
stored bytes of every logit, and the bytes verification needs given the
accepted lengths (rows after a request's first rejection, or off a tree's
accepted path, are not needed)."""
import numpy as np
import torch

import bench
from speculative_decoding_verification_94_b200 import inputs


def _nbytes(*ts):
    return sum(t.numel() * t.element_size() for t in ts)


def test_chain_stored_and_needed_bytes():
    x = inputs.make_chain(3, 3, 257, dtype="bf16", seed=1)
    rows, full = bench.rows_and_bytes("chain", x)
    assert rows == 3 * 4
    io = _nbytes(x.draft_tokens, x.uniforms) + 3 * 4 + 3 * 4 * 4  # accepted_len, out_tokens
    assert full == _nbytes(x.target, x.draft) + io
    acc = np.array([0, 2, 3], np.int32)
    # request 0: pair 0; request 1: pairs 0..2; request 2: pairs 0..2 and the bonus row 3
    pair = 257 * 2 * 2
    want = (1 + 3 + 3) * pair + 257 * 2 + io
    assert bench.needed_bytes("chain", x, acc) == want


def test_sampling_tree_bytes_count_visited_nodes():
    t = inputs.make_tree_sample(B=2, V=300, depth_counts=(2, 2), branching=2, seed=2)
    B, n, V = t.target.shape
    rows, full = bench.rows_and_bytes("tree_sample", t)
    assert rows == B * n
    small = _nbytes(t.node_tokens, t.parents, t.uniforms) + B * 4 + 2 * B * (t.max_depth + 1) * 4
    assert full == _nbytes(t.target, t.draft) + small
    acc = np.array([2, 0], np.int32)  # visits: root..depth 2 (3 nodes), root only (1 node)
    assert bench.needed_bytes("tree_sample", t, acc) == 4 * V * (2 + 2) + small


def test_greedy_tree_reads_every_node():
    t = inputs.make_tree(B=2, V=300, depth_counts=(2, 2), branching=2, seed=3)
    rows, full = bench.rows_and_bytes("tree", t)
    assert rows == 2 * t.logits.shape[1]
    assert bench.needed_bytes("tree", t, np.zeros(2, np.int32)) == full
    assert full >= _nbytes(t.logits)


def test_job_value_is_whole_job_rows_per_second():
    # 2 ranks x 10 steps x 128 rows in 5 ms of the slowest rank
    assert bench.job_value(128, 2, 10, 5.0) == 128 * 2 * 10 / 5e-3


def test_ragged_bytes_count_only_used_rows():
    x = inputs.make_chain(4, 3, 300, dtype="bf16", seed=4)
    x.meta["draft_len"] = torch.tensor([0, 3, 2, 1], dtype=torch.int32)
    x.meta["active"] = torch.tensor([1, 1, 0, 1], dtype=torch.int32)
    rows, full = bench.rows_and_bytes("ragged", x)
    assert rows == 1 + 4 + 2  # idle request 2 uses no row
    io = _nbytes(x.draft_tokens, x.uniforms) + 2 * 4 * 4 + 4 * 4 + 4 * 4 * 4
    row = 300 * 2
    assert full == (7 * row + (0 + 3 + 1) * row) + io
    acc = np.array([0, 1, 0, 1], np.int32)
    # request 0: bonus row 0; request 1: pairs 0..1; request 3: pair 0 and bonus row 1
    assert bench.needed_bytes("ragged", x, acc) == (0 + 2 + 1) * 2 * row + 2 * row + io


def test_ragged_lengths_cover_every_length():
    kl, act = inputs.ragged_lengths(32, 3, seed=0)
    assert kl.dtype == torch.int32 and act.dtype == torch.int32
    assert set(kl.tolist()) == {0, 1, 2, 3} and (act[:4] == 1).all()
    assert ((kl >= 0) & (kl <= 3)).all() and 0 < int(act.sum()) <= 32


def test_dominant_kernel_and_its_bytes():
    """The roofline's kernel: the streaming pass carries every logit of a chain
    or greedy tree; the gradient kernel carries all but the statistics pass's
    read of the draft rows; a sampling tree or a persistent call has one
    kernel."""
    x = inputs.make_chain(3, 3, 257, dtype="bf16", seed=1)
    _, full = bench.rows_and_bytes("chain", x)
    two = {"stream_kernel": {}, "chain_sample_finish": {}}
    assert bench.dominant_kernel("chain", x, full, two) == ("stream_kernel", full)
    assert bench.dominant_kernel("chain", x, full, {"chain_kernel": {}}) == ("chain_kernel", full)
    _, gfull = bench.rows_and_bytes("grad", x)
    name, by = bench.dominant_kernel("grad", x, gfull, {"stream_kernel": {}, "kd_grad_kernel": {}})
    assert name == "kd_grad_kernel"
    assert by == gfull - _nbytes(x.draft)
    assert bench.kernel_names("tree")["finish"] == "tree_finish"
    assert bench.kernel_names("kd")["stream"] == "stream_kernel"


def test_peaks_fallback_and_file(tmp_path, monkeypatch):
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    assert bench.load_peaks() == (6650.0, "fallback")
    (tmp_path / "MEASURED_PEAKS.json").write_text('{"hbm_gbs": 6545.3, "bf16_tflops": 1590}')
    assert bench.load_peaks() == (6545.3, "measured")
    (tmp_path / "MEASURED_PEAKS.json").write_text('{"HBM_copy_GBps": 6400}')
    assert bench.load_peaks() == (6400.0, "measured")
