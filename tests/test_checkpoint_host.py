"""Checkpoint host logic on CPU tensors: a snapshot restores in place, bit for
bit, and refuses a run of another kind or other shapes."""
import os

import pytest
import torch

from matrix_aware_sign_b200 import checkpoint as C


def test_snapshot_restores_in_place(tmp_path):
    g = torch.Generator().manual_seed(0)
    state = {"W": torch.randn(7, 9, generator=g), "m": torch.randn(3, 5, generator=g).to(torch.bfloat16)}
    keep = {k: v.data_ptr() for k, v in state.items()}
    path = os.path.join(tmp_path, "ck.pt")
    C.save(path, state)
    want = {k: v.clone() for k, v in state.items()}
    for v in state.values():
        v.add_(1)
    C.load(path, state)
    for k in state:
        assert torch.equal(state[k], want[k]) and state[k].data_ptr() == keep[k]


def test_restore_refuses_a_different_run():
    snap = C.snapshot({"W": torch.zeros(4, 4)})
    with pytest.raises(ValueError):
        C.restore({"W": torch.zeros(4, 5)}, snap)
    with pytest.raises(ValueError):
        C.restore({"V": torch.zeros(4, 4)}, snap)
    with pytest.raises(ValueError):
        C.restore({"W": torch.zeros(4, 4, dtype=torch.float64)}, snap)
    with pytest.raises(TypeError):
        C.snapshot([torch.zeros(1)])
