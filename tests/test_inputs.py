"""The stored redraw tables are exactly what the oracle's margin screen gives
for the seeded generator, so every stored workload has a unique top-k."""
import pytest

import synth
from tests.golden import make_redraws


@pytest.mark.parametrize("name", list(make_redraws.JOBS))
def test_redraw_table_reproduces(name):
    for T, steps in make_redraws.JOBS[name]:
        stored = synth.load_redraws(name, T)
        assert stored is not None, f"missing {synth.redraw_path(name, T)}"
        assert make_redraws.screen(name, T, steps) == stored


def test_generator_is_deterministic_and_counter_addressed():
    a = synth.normal(0, synth.TAG_EXPERT, 3, 1, 0, 1000, 0.02)
    b = synth.normal(0, synth.TAG_EXPERT, 3, 1, 0, 2000, 0.02)
    assert (a == b[:1000]).all()
    c = synth.normal(0, synth.TAG_EXPERT, 3, 2, 0, 1000, 0.02)
    assert not (a == c).all()
    p = synth.permutation(0, synth.TAG_SLOTS, 128)
    assert sorted(p.tolist()) == list(range(128))
