"""The Python binding only marshals arguments: it refuses host tensors for
every device entry point (there is no CPU fallback), and it raises when the
CUDA library is missing instead of computing anything itself."""
from pathlib import Path

import pytest
import torch

from speculative_decoding_verification_94_b200 import sv


def test_device_entry_points_refuse_host_tensors():
    z = torch.zeros(2, 4, 64, dtype=torch.bfloat16)
    d = torch.zeros(2, 3, 64, dtype=torch.bfloat16)
    tok = torch.zeros(2, 3, dtype=torch.int32)
    u = torch.zeros(2, 4)
    calls = [
        lambda: sv.sv_verify_chain(z, d, tok, u, 0.7),
        lambda: sv.sv_verify_chain_ragged(z, d, tok, u, 0.7,
                                          draft_len=torch.zeros(2, dtype=torch.int32)),
        lambda: sv.sv_verify_chain_noalloc(z, d, tok, u, 0.7),
        lambda: sv.sv_verify_tree_greedy(z, torch.zeros(2, 4, dtype=torch.int32),
                                         torch.zeros(2, 4, dtype=torch.int32), 2),
        lambda: sv.sv_verify_tree_sample(z, z, torch.zeros(2, 4, dtype=torch.int32),
                                         torch.zeros(2, 4, dtype=torch.int32), u, 0.7, 2),
        lambda: sv.sv_extract_topk_kd(z, 8, 0.7),
    ]
    for call in calls:
        with pytest.raises(TypeError, match="CUDA tensor"):
            call()


def test_missing_library_raises(monkeypatch):
    monkeypatch.setattr(sv, "_LIB_PATH", Path("/nonexistent/libsv.so"))
    monkeypatch.setattr(sv, "_lib", None)
    with pytest.raises(RuntimeError, match="missing"):
        sv.lib()
