"""The C ABI library loads and exports every function include/sv.h declares;
host-side validation rejects bad arguments before any CUDA call (so these run
without a GPU)."""
import ctypes
import os
import re
import subprocess

import pytest

from speculative_decoding_verification_94_b200 import sv

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "sv.h")


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"^[A-Za-z_][\w \*]*?\b(sv_\w+)\s*\(", text, flags=re.M)))


@pytest.fixture(scope="module")
def lib():
    from speculative_decoding_verification_94_b200 import build
    build.build()
    return sv.lib()


def test_header_declares_the_entry_points():
    names = declared_functions()
    for f in ("sv_verify_chain", "sv_verify_tree_greedy", "sv_extract_topk_kd", "sv_kd_kl_loss"):
        assert f in names
    assert set(names) == set(sv.EXPORTS)


def test_library_exports_every_declared_symbol(lib):
    for name in declared_functions():
        assert hasattr(lib, name), name
    out = subprocess.run(["nm", "-D", "--defined-only", str(sv.lib_path())], capture_output=True,
                         text=True, check=True).stdout
    exported = {line.split()[-1] for line in out.splitlines() if line.strip()}
    assert set(declared_functions()) <= exported
    # nothing else of ours leaks out of the shared object
    assert not [s for s in exported if s.startswith("sv_") and s not in sv.EXPORTS]


def test_status_strings_and_version(lib):
    assert sv.status_string(0) == "ok"
    assert "workspace" in sv.status_string(6)
    assert sv.sv_version() >= 100
    assert sv.sv_device_status_check(0) == sv.SV_OK
    assert sv.sv_device_status_check(sv.SV_DEV_RESIDUAL_ZERO | sv.SV_DEV_TOPK_SLOW) == sv.SV_OK
    assert sv.sv_device_status_check(sv.SV_DEV_BAD_TOKEN) == sv.SV_ERR_DEVICE_CHECK
    assert sv.sv_device_status_check(sv.SV_DEV_TIMEOUT | 1) == sv.SV_ERR_TIMEOUT


def test_workspace_sizes(lib):
    assert sv.sv_verify_chain_workspace_size(0, 3, 1024) == 256
    V = 151936
    a = sv.sv_verify_chain_workspace_size(32, 3, V)
    nchunk = -(-V // 8192)
    # records, partials and counters of 128 rows; KD adds K keys per chunk
    assert a % 256 == 0 and a >= 128 * (48 + 48 * nchunk + 4) + 4 * 32
    assert sv.sv_verify_chain_workspace_size(32, 3, V, 32) >= a + 128 * nchunk * 32 * 8
    assert sv.sv_verify_tree_workspace_size(8, 32, V) >= 256 * 48 * nchunk
    assert sv.sv_extract_topk_workspace_size(10, 1000, 32) >= 10 * (48 + 48 + 32 * 8)
    assert sv.sv_kd_kl_loss_workspace_size(256, 3, V) >= 768 * 48 * nchunk


FAKE = ctypes.c_void_p(0x10000)  # never dereferenced: every call below fails validation

# The calls below hand fake device addresses to the library and expect host
# validation to reject them.  They run only where no GPU is present, so that a
# validation gap can never turn into a kernel launch on bogus addresses.
no_gpu = pytest.mark.skipif(__import__("torch").cuda.is_available(),
                            reason="fake-pointer validation tests run only without a GPU")


def _chain(lib, **kw):
    a = dict(target=FAKE, tdt=sv.SV_BF16, draft=FAKE, ddt=sv.SV_BF16, dk=sv.SV_DRAFT_LOGITS,
             tok=FAKE, u=FAKE, B=4, k=3, V=1024, T=1.0, acc=FAKE, out=FAKE, kd=None, ws=FAKE,
             wsb=1 << 20, status=None, stream=None)
    a.update(kw)
    return lib.sv_verify_chain(a["target"], a["tdt"], a["draft"], a["ddt"], a["dk"], a["tok"],
                               a["u"], a["B"], a["k"], a["V"], a["T"], a["acc"], a["out"],
                               a["kd"], a["ws"], a["wsb"], a["status"], a["stream"])


@no_gpu
def test_chain_validation_rejects_before_any_cuda_call(lib):
    E = sv.SV_ERR_INVALID_ARG
    assert _chain(lib, target=None) == E
    assert _chain(lib, k=0) == E
    assert _chain(lib, k=256) == E
    assert _chain(lib, V=0) == E
    assert _chain(lib, B=-1) == E
    assert _chain(lib, T=-1.0) == E
    assert _chain(lib, T=float("nan")) == E
    assert _chain(lib, T=float("inf")) == E
    assert _chain(lib, T=1e-45) == E  # 1/T overflows
    assert _chain(lib, tdt=7) == E
    assert _chain(lib, draft=None) == E
    assert _chain(lib, u=None) == E
    assert _chain(lib, dk=sv.SV_DRAFT_PROBS, ddt=sv.SV_BF16) == E
    assert _chain(lib, tok=ctypes.c_void_p(0x10002)) == E  # misaligned int32
    kd = sv.sv_kd_args(0, 0x10000, 0x10000, 0x10000, 0x10000, 0x10000, 0, 1, 0.0, 0x10000, 0x10000)
    assert _chain(lib, kd=ctypes.byref(kd)) == E  # K = 0
    kd.K = 32
    assert _chain(lib, kd=ctypes.byref(kd), T=0.0) == E  # KD needs T > 0
    kd.wmode, kd.group = sv.SV_W_GROUP_NORM, 3
    assert _chain(lib, kd=ctypes.byref(kd)) == E  # B % group != 0
    assert _chain(lib, ws=None) == sv.SV_ERR_WORKSPACE
    assert _chain(lib, wsb=16) == sv.SV_ERR_WORKSPACE
    assert _chain(lib, ws=ctypes.c_void_p(0x10004)) == sv.SV_ERR_WORKSPACE
    assert _chain(lib, V=600000, wsb=1 << 40) == sv.SV_ERR_UNSUPPORTED
    # empty batch: nothing to do, nothing enqueued
    assert _chain(lib, B=0, ws=None) == sv.SV_OK
    # greedy: draft and uniforms may be NULL (fails only on the workspace here)
    assert _chain(lib, T=0.0, draft=None, u=None, ws=None) == sv.SV_ERR_WORKSPACE


@no_gpu
def test_other_entry_points_validate(lib):
    E = sv.SV_ERR_INVALID_ARG
    f = FAKE
    # tree: parents NULL, n too large, max_depth >= n
    assert lib.sv_verify_tree_greedy(f, 1, f, None, 2, 32, 100, 5, f, f, f, f, 1 << 20, None,
                                     None) == E
    assert lib.sv_verify_tree_greedy(f, 1, f, f, 2, 2000, 100, 5, f, f, f, f, 1 << 20, None,
                                     None) == E
    assert lib.sv_verify_tree_greedy(f, 1, f, f, 2, 4, 100, 4, f, f, f, f, 1 << 20, None,
                                     None) == E
    # top-K: K > 32, K > V, T == 0
    assert lib.sv_extract_topk_kd(f, 1, 4, 1000, 33, 1.0, f, f, f, f, 1 << 20, None, None) == E
    assert lib.sv_extract_topk_kd(f, 1, 4, 10, 16, 1.0, f, f, f, f, 1 << 20, None, None) == E
    assert lib.sv_extract_topk_kd(f, 1, 4, 1000, 32, 0.0, f, f, f, f, 1 << 20, None, None) == E
    assert lib.sv_extract_topk_kd(f, 1, 0, 1000, 32, 1.0, f, f, f, f, 1 << 20, None,
                                  None) == sv.SV_OK
    assert lib.sv_extract_topk_kd(f, 1, 4, 1000, 32, 1.0, f, f, f, f, 16, None,
                                  None) == sv.SV_ERR_WORKSPACE
    # KL loss: probs must be fp32, group must divide B
    assert lib.sv_kd_kl_loss(f, f, 4, 3, 32, f, sv.SV_BF16, sv.SV_DRAFT_PROBS, 1000, 1.0, f, f,
                             0, 1, 0.0, 0, f, f, f, f, 1 << 20, None, None) == E
    assert lib.sv_kd_kl_loss(f, f, 4, 3, 32, f, sv.SV_BF16, sv.SV_DRAFT_LOGITS, 1000, 1.0, f, f,
                             1, 3, 0.0, 0, f, f, f, f, 1 << 20, None, None) == E
    assert lib.sv_kd_kl_loss(f, f, 4, 3, 32, f, sv.SV_BF16, sv.SV_DRAFT_LOGITS, 1000, 1.0, f, f,
                             0, 1, 0.0, 0, f, f, f, None, 1 << 20, None, None) == sv.SV_ERR_WORKSPACE


@no_gpu
def test_ragged_chain_and_sampling_tree_validate(lib):
    E = sv.SV_ERR_INVALID_ARG
    f = FAKE

    def ragged(dl, act, ws=f):
        return lib.sv_verify_chain_ragged(f, sv.SV_BF16, f, sv.SV_BF16, sv.SV_DRAFT_LOGITS, f, f,
                                          dl, act, 4, 3, 1024, 1.0, f, f, None, ws, 1 << 20,
                                          None, None)
    assert ragged(ctypes.c_void_p(0x10002), None) == E  # misaligned draft_len
    assert ragged(None, ctypes.c_void_p(0x10001)) == E  # misaligned active
    assert ragged(f, f, ws=None) == sv.SV_ERR_WORKSPACE  # arrays fine, fails on the workspace

    def tree(**kw):
        a = dict(t=f, tdt=sv.SV_BF16, d=f, ddt=sv.SV_BF16, dk=sv.SV_DRAFT_LOGITS, tok=f, par=f,
                 u=f, B=4, n=32, V=1024, depth=5, T=0.7, acc=f, out=f, nodes=f)
        a.update(kw)
        return lib.sv_verify_tree_sample(a["t"], a["tdt"], a["d"], a["ddt"], a["dk"], a["tok"],
                                         a["par"], a["u"], a["B"], a["n"], a["V"], a["depth"],
                                         a["T"], a["acc"], a["out"], a["nodes"], None, None)
    assert tree(T=0.0) == E                      # sampling needs T > 0
    assert tree(n=0) == E
    assert tree(n=2000) == E
    assert tree(depth=32) == E                   # max_depth >= n
    assert tree(dk=sv.SV_DRAFT_PROBS) == E       # probabilities must be fp32
    assert tree(u=None) == E
    assert tree(par=None) == E
    assert tree(d=ctypes.c_void_p(0x10001)) == E  # misaligned bf16 row
    assert tree(V=600000) == sv.SV_ERR_UNSUPPORTED
    assert tree(B=0) == sv.SV_OK                 # nothing to do, nothing enqueued


def _noalloc(lib, **kw):
    a = dict(target=FAKE, tdt=sv.SV_BF16, draft=FAKE, ddt=sv.SV_BF16, dk=sv.SV_DRAFT_LOGITS,
             tok=FAKE, u=FAKE, B=4, k=3, V=1024, T=1.0, acc=FAKE, out=FAKE, kd=None,
             status=None, stream=None)
    a.update(kw)
    return lib.sv_verify_chain_noalloc(a["target"], a["tdt"], a["draft"], a["ddt"], a["dk"],
                                       a["tok"], a["u"], a["B"], a["k"], a["V"], a["T"],
                                       a["acc"], a["out"], a["kd"], a["status"], a["stream"])


@no_gpu
def test_noalloc_checks_arguments_like_the_workspace_call(lib):
    """Bad arguments give sv_verify_chain's code, not a scratch-size error,
    even where the declared sizes would also overflow the fixed scratch."""
    big = dict(B=4096, V=151936)
    kd = sv.sv_kd_args(1000, 0x10000, 0x10000, 0x10000, 0x10000, 0x10000, 0, 1, 0.0, 0x10000,
                       0x10000)
    for kw in (dict(kd=ctypes.byref(kd)), dict(k=300), dict(k=0), dict(T=-1.0),
               dict(dk=sv.SV_DRAFT_PROBS, ddt=sv.SV_BF16), dict(V=600000)):
        args = dict(big, **kw)
        want = _chain(lib, wsb=1 << 40, **args)
        assert want != sv.SV_OK
        assert _noalloc(lib, **args) == want, kw
    # valid arguments beyond the scratch: the size check answers
    assert _noalloc(lib, **big) == sv.SV_ERR_WORKSPACE
    assert _noalloc(lib, B=0) == sv.SV_OK


def test_knobs_validate(lib):
    assert lib.sv_set_knob(0, 1) == sv.SV_ERR_INVALID_ARG
    assert lib.sv_set_knob(99, 1) == sv.SV_ERR_INVALID_ARG
    assert lib.sv_set_knob(sv.SV_KNOB_STAGES, 0) == sv.SV_OK
    assert lib.sv_set_knob(sv.SV_KNOB_FINISH_READ + 1, 1) == sv.SV_ERR_INVALID_ARG


def test_kernel_times_without_marks(lib):
    """No marked launch yet: zero launches reported, no device touched; null
    pointers are refused."""
    import ctypes
    n = ctypes.c_int32(7)
    us = (ctypes.c_float * 4)()
    tags = (ctypes.c_int32 * 4)()
    assert lib.sv_kernel_times(us, tags, 4, ctypes.byref(n)) == sv.SV_OK
    assert n.value == 0
    assert lib.sv_kernel_times(us, tags, 4, None) == sv.SV_ERR_INVALID_ARG
    assert lib.sv_kernel_times(None, None, 4, ctypes.byref(n)) == sv.SV_ERR_INVALID_ARG
