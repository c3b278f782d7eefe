"""The randomised round trip of the expert-parallel exchange plan catches plausible
slips: each change below, planted in an in-memory copy of ``exchange_plan`` (the
module's file is untouched), makes the whole-world round trip fail."""
import inspect

import pytest

from sparse_mixture_experts_09_b200 import ep

from . import test_ep as T

MUTATIONS = [
    # received segments ordered expert-major instead of by source rank
    ("    for s in range(world):\n        for e in range(e_loc):\n            seg[s][e] = pos",
     "    for e in range(e_loc):\n        for s in range(world):\n            seg[s][e] = pos"),
    # local groups gathered source-major instead of expert-major
    ("    for e in range(e_loc):\n        for s in range(world):\n            to_local.extend",
     "    for s in range(world):\n        for e in range(e_loc):\n            to_local.extend"),
    # rows sent to a rank counted over the wrong experts
    ("send_rows = [sum(counts[r * e_loc:(r + 1) * e_loc]) for r in range(world)]",
     "send_rows = [sum(counts[r:r + e_loc]) for r in range(world)]"),
    # pad rows sent along with the real ones
    ("        for j in range(counts[e]):", "        for j in range(offsets[e + 1] - offsets[e]):"),
    # local groups not padded to whole tiles
    ("        to_local.extend([-1] * (_pad(len(to_local) - local_offsets[-1]) -",
     "        to_local.extend([-1] * (0 * _pad(len(to_local) - local_offsets[-1]) -"),
]


@pytest.mark.parametrize("old,new", MUTATIONS, ids=[f"m{i}" for i in range(len(MUTATIONS))])
def test_planted_plan_mistake_fails_the_round_trip(monkeypatch, old, new):
    src = inspect.getsource(ep.exchange_plan)
    assert src.count(old) == 1, f"the planted text must occur once: {old!r}"
    ns = {}
    exec(compile(src.replace(old, new), ep.__file__, "exec"), ep.__dict__.copy(), ns)
    monkeypatch.setattr(T.ep, "exchange_plan", ns["exchange_plan"])
    with pytest.raises((AssertionError, IndexError, ValueError)):
        T.test_exchange_plan_random_worlds_round_trip()


def test_unplanted_plan_passes():
    T.test_exchange_plan_random_worlds_round_trip()
