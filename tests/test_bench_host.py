"""Host-side rules of bench.py's timing that need no GPU."""
import sys

from conftest import ROOT

sys.path.insert(0, ROOT)

import bench  # noqa: E402


def test_warmup_covers_whole_rotations():
    # the requested warm-up, rounded up to whole passes over the layer buffers
    assert bench.warmup_pass_steps(3, 29) == 29
    assert bench.warmup_pass_steps(29, 29) == 29
    assert bench.warmup_pass_steps(30, 29) == 58
    assert bench.warmup_pass_steps(50, 29) == 58
    # one buffer: exactly the requested steps; never an empty pass
    assert bench.warmup_pass_steps(3, 1) == 3
    assert bench.warmup_pass_steps(0, 1) == 1
    assert bench.warmup_pass_steps(0, 0) == 1


def test_warmup_lasts_long_enough_for_a_steady_state():
    assert bench.WARM_MIN_S >= 0.05
