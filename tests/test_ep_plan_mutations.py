"""The randomised round trip of the expert-parallel exchange plan catches plausible
slips: each change below, planted in an in-memory copy of ``exchange_plan`` (the
module's file is untouched), makes the whole-world round trip fail."""
import inspect

import pytest

from sparse_mixture_experts_09_b200 import ep

from . import test_ep as T

MUTATIONS = [
    # received segments ordered expert-major instead of by source rank
    ("seg_start = _starts(rc.reshape(-1)).reshape(world, e_loc)",
     "seg_start = _starts(rc.t().reshape(-1)).reshape(e_loc, world).t()"),
    # sources of a local group in reverse order
    ("before = (torch.cumsum(rc, 0) - rc).t()",
     "before = (torch.cumsum(rc.flip(0), 0) - rc.flip(0)).flip(0).t()"),
    # rows sent to a rank counted over the wrong experts
    ("send_rows = counts_h.reshape(world, e_loc).sum(1).tolist()",
     "send_rows = counts_h.reshape(e_loc, world).sum(0).tolist()"),
    # pad rows sent along with the real ones
    ("grp, j = _segment_ranks(counts, n_send)",
     "grp, j = _segment_ranks(offsets[1:] - offsets[:-1], n_rows)"),
    # local groups not padded to whole tiles
    ("local_offsets = [0] + torch.cumsum(_pad(rc_h.sum(0)), 0).tolist()",
     "local_offsets = [0] + torch.cumsum(rc_h.sum(0), 0).tolist()"),
]


@pytest.mark.parametrize("old,new", MUTATIONS, ids=[f"m{i}" for i in range(len(MUTATIONS))])
def test_planted_plan_mistake_fails_the_round_trip(monkeypatch, old, new):
    src = inspect.getsource(ep.exchange_plan)
    assert src.count(old) == 1, f"the planted text must occur once: {old!r}"
    ns = {}
    exec(compile(src.replace(old, new), ep.__file__, "exec"), ep.__dict__.copy(), ns)
    monkeypatch.setattr(T.ep, "exchange_plan", ns["exchange_plan"])
    with pytest.raises((AssertionError, IndexError, ValueError, RuntimeError)):
        T.test_exchange_plan_random_worlds_round_trip()


def test_unplanted_plan_passes():
    T.test_exchange_plan_random_worlds_round_trip()
