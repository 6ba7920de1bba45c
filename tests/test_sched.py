"""The adaptive scheduler lookup (host code, no GPU): the oracle against the
pages' worked example and numpy's interpolation, and sv_sched_select through
the C ABI against the oracle."""
import json
import os

import numpy as np
import pytest

from oracle import oracle as O

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _golden():
    with open(os.path.join(GOLDEN, "respec_scheduler_example.json"), encoding="utf-8") as f:
        return json.load(f)


def _tables(seed, n=200):
    rng = np.random.default_rng(seed)
    for _ in range(n):
        n_cfg = int(rng.integers(1, 7))
        nb = int(rng.integers(1, 8))
        bs = np.sort(rng.choice(np.arange(1, 129), nb, replace=False)).astype(np.int32)
        thr = rng.uniform(0.2, 2.0, (n_cfg, nb)).astype(np.float32)
        if rng.random() < 0.2 and n_cfg > 2:
            thr[2] = thr[1]  # a tie between two speculative rows
        nonspec = int(rng.integers(0, n_cfg))
        thr[nonspec] = rng.uniform(0.5, 1.5, nb).astype(np.float32)
        yield thr, bs, nonspec, int(rng.integers(1, 160))


def test_scheduler_worked_example(oracle):
    g = _golden()
    for e in g["expect"]:
        cfg, sp = oracle.sched_select(g["throughput"], g["batches"], g["nonspec"],
                                      e["active_batch"])
        assert cfg == e["config"]
        if "speedup" in e:
            assert sp == pytest.approx(e["speedup"], rel=1e-6)


def test_scheduler_matches_numpy_interp(oracle):
    """Each row's lookup is numpy.interp in the batch size; the choice is the
    best speculative row unless it is slower than plain decoding."""
    for thr, bs, nonspec, a in _tables(1):
        cfg, sp = oracle.sched_select(thr, bs, nonspec, a)
        vals = np.array([np.interp(a, bs, row.astype(np.float64)) for row in thr])
        spec = [c for c in range(len(thr)) if c != nonspec]
        if not spec:
            assert cfg == nonspec and sp == 0.0
            continue
        best = spec[int(np.argmax(vals[spec]))]  # first maximum: lowest index
        want_sp = vals[best] / vals[nonspec]
        assert sp == pytest.approx(want_sp, rel=1e-12)
        assert cfg == (best if want_sp >= 1.0 else nonspec) or abs(want_sp - 1.0) < 1e-12


def test_sched_select_abi_matches_oracle(oracle):
    from speculative_decoding_verification_94_b200 import sv
    for thr, bs, nonspec, a in _tables(2, n=400):
        cfg, sp = sv.sv_sched_select(thr, bs, nonspec, a)
        ocfg, osp = oracle.sched_select(thr, bs, nonspec, a)
        assert cfg == ocfg
        assert sp == pytest.approx(osp, rel=1e-6)
    g = _golden()
    for e in g["expect"]:
        cfg, _ = sv.sv_sched_select(g["throughput"], g["batches"], g["nonspec"], e["active_batch"])
        assert cfg == e["config"]


def test_sched_select_rejects_bad_tables():
    from speculative_decoding_verification_94_b200 import sv
    ok = np.ones((2, 3), np.float32)
    bs = np.array([1, 4, 16], np.int32)
    assert sv.sv_sched_select(ok, bs, 0, 5)[0] in (0, 1)
    bad = [
        (ok, np.array([1, 4, 4], np.int32), 0, 5),   # not strictly ascending
        (ok, np.array([0, 4, 16], np.int32), 0, 5),  # batch < 1
        (ok, bs, 2, 5),                               # nonspec out of range
        (ok, bs, 0, 0),                               # no active request
        (np.array([[0, 1, 1], [1, 1, 1]], np.float32), bs, 0, 1),  # zero plain throughput
        (np.array([[1, 1, 1], [1, np.nan, 1]], np.float32), bs, 0, 5),
        (np.array([[1, 1, 1], [-1, 1, 1]], np.float32), bs, 0, 5),
    ]
    for thr, b, ns, a in bad:
        with pytest.raises(RuntimeError):
            sv.sv_sched_select(thr, b, ns, a)


TABLE = os.path.join(os.path.dirname(os.path.dirname(__file__)),
                     "speculative_decoding_verification_94_b200", "data", "verify_cost_table.json")


def test_sched_select_on_the_measured_verify_cost_table(oracle):
    """The lookup over the measured verify-kernel cost table of this device
    (emitted tokens per second of one verification call for plain decoding
    and k = 1, 3, 5, 7 drafts at active batches 1..32, written by
    `bench.py --workload sched_table`): the C ABI's choice and predicted
    speedup equal the oracle's at every active batch, inside and outside the
    profiled sizes."""
    from speculative_decoding_verification_94_b200 import sv
    with open(TABLE, encoding="utf-8") as f:
        t = json.load(f)
    thr = np.asarray(t["throughput_tokens_per_s"], np.float32)
    bs = np.asarray(t["batches"], np.int32)
    assert thr.shape == (len(t["configs"]), len(bs)) and (thr > 0).all()
    chosen = []
    for a in range(1, 65):
        cfg, sp = sv.sv_sched_select(thr, bs, t["nonspec"], a)
        ocfg, osp = oracle.sched_select(thr, bs, t["nonspec"], a)
        assert cfg == ocfg, a
        assert sp == pytest.approx(osp, rel=1e-6), a
        chosen.append(t["configs"][cfg])
    print("configuration per active batch 1..64:", chosen)
