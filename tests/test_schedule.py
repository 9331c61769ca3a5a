"""Host logic of the cross-step mask reuse schedule (MOD-DiT: warm-up steps
of full attention, then a pattern refreshed every delta-t steps;
HyperVAttention section 3: selections stable across adjacent steps)."""
import pytest

from block_sparse_attention_pool_b200 import SelectionSchedule


def test_warmup_then_refresh_period():
    s = SelectionSchedule(warmup=2, refresh=3)
    assert [s.mode(t) for t in range(9)] == ["dense", "dense", "select", "reuse", "reuse", "select", "reuse",
                                              "reuse", "select"]


def test_refresh_every_step_never_reuses():
    s = SelectionSchedule(warmup=0, refresh=1)
    assert {s.mode(t) for t in range(20)} == {"select"}


def test_first_sparse_step_always_selects():
    for w in range(4):
        for r in range(1, 5):
            s = SelectionSchedule(w, r)
            assert s.mode(w) == "select"
            # exactly one selection per period after the warm-up
            modes = [s.mode(t) for t in range(w, w + 4 * r)]
            assert modes.count("select") == 4


@pytest.mark.parametrize("args", [(-1, 2), (0, 0)])
def test_invalid_schedule(args):
    with pytest.raises(ValueError):
        SelectionSchedule(*args)
    with pytest.raises(ValueError):
        SelectionSchedule().mode(-1)
