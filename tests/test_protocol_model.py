"""The attention kernel's mbarrier hand-offs, checked on an executable model.

tests/protocol_model.py replays the kernel's roles (producers, QK^T and P.V
issuers, twelve softmax warps) with the ring sizes the kernel uses, under
random schedules, random completion delays and random BF16 tile patterns,
and fails on any parity wait that could pass early or never return, and on
deadlock.  The same model with the rings the kernel's comments argue against
(two S_FULL barriers for three groups, four P.V completion barriers, one P_FULL
slot per group) must fail, which shows the check can see the hazards it rules
out.
"""
import random

import pytest

from protocol_model import Model, ProtocolError, Rings


def _patterns(n, seed):
    rng = random.Random(seed)
    for trial in range(n):
        nj = rng.randint(1, 70)
        p = rng.choice([0.0, 0.05, 0.25, 0.6, 1.0])
        hi = [rng.random() < p for _ in range(nj)]
        hi[0] = True            # sink tile
        hi[-1] = True           # diagonal tile
        yield trial, hi


def test_committed_rings_are_sound_under_random_schedules():
    for trial, hi in _patterns(160, seed=1):
        Model(hi, rings=Rings(), seed=trial).run()


def test_long_rows_with_runs_of_bf16_tiles():
    rng = random.Random(2)
    for trial in range(12):
        hi = [False] * 200
        for start in rng.sample(range(200), 12):
            for j in range(start, min(200, start + rng.randint(1, 4))):
                hi[j] = True
        hi[0] = hi[-1] = True
        Model(hi, rings=Rings(), seed=100 + trial).run()


@pytest.mark.parametrize("rings", [Rings(s_full=2), Rings(pvc=4), Rings(p_ring=1)],
                         ids=["two S_FULL barriers", "four P.V completion barriers", "one P_FULL slot"])
def test_undersized_rings_are_caught(rings):
    with pytest.raises(ProtocolError):
        for trial, hi in _patterns(300, seed=1):
            Model(hi, rings=rings, seed=trial).run()
