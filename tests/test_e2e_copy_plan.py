"""Host check (no GPU) of the pipelined end-to-end step's copy plan: every
layer's input is copied in exactly once and its output out exactly once, and
the copies cover the layers in order."""
import importlib.util
import os

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _bench():
    spec = importlib.util.spec_from_file_location("bench_under_test", os.path.join(ROOT, "bench.py"))
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    return mod


@pytest.mark.parametrize("L", [1, 2, 3, 4, 5, 8, 48, 64])
def test_copies_cover_every_layer_once(L):
    in_cuts, out_cuts = _bench().e2e_copy_cuts(L)
    for cuts in (in_cuts, out_cuts):
        assert cuts[0] == 0 and cuts[-1] == L
        assert all(a < b for a, b in zip(cuts[:-1], cuts[1:])), cuts
        covered = [l for a, b in zip(cuts[:-1], cuts[1:]) for l in range(a, b)]
        assert covered == list(range(L))
    # at most one wait between layers on the input side, two output copies
    assert len(in_cuts) - 1 <= 2 and len(out_cuts) - 1 <= 2
    if L > 4:
        assert in_cuts[1] == 4 and out_cuts[1] == L - 4
