"""The clip schedule against the pages' Tables 3 and 4, and the renoise oracle's closed forms."""
import os
from fractions import Fraction

import numpy as np
import pytest
import torch

import oracle
from causal_video_diffusion_b200 import schedule as S
from causal_video_diffusion_b200 import workloads as W

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _table4():
    rows, clean = [], {}
    for line in open(os.path.join(GOLDEN, "table4_shift5_schedule.txt")):
        line = line.strip()
        if not line or line.startswith("#"):
            continue
        parts = line.split()
        if parts[0].startswith("clean"):
            clean[parts[0]] = (float(parts[1]), float(parts[2]))
        else:
            rows.append((int(parts[0]), int(parts[1]), Fraction(int(parts[2]), int(parts[3])),
                         float(parts[4])))
    return rows, clean


def test_shift5_mapping_reproduces_table4():
    rows, clean = _table4()
    for i, u, sig, label in rows:
        assert S.FOUR_STEPS[i] == u
        # the mapping in exact rationals: 5 u' / (1 + 4 u')
        x = Fraction(u, 1000)
        assert 5 * x / (1 + 4 * x) == sig
        assert S.shifted_sigma(u) == pytest.approx(float(sig), abs=1e-15)
        assert 1000 * S.shifted_sigma(u) == pytest.approx(label, abs=0.05)   # table rounds to 0.1
    assert clean["clean_sf"] == (S.CLEAN_SIGMA["self_forcing"], 0.0)
    assert clean["clean_unstep"] == (S.CLEAN_SIGMA["unstep"], 0.0)


def test_clip_schedules_match_table3():
    assert len(S.clip_schedule("unstep")) == 23
    assert len(S.clip_schedule("self_forcing")) == 35
    assert S.forwards_per_chunk("unstep") == W.UNSTEP_FORWARDS
    assert S.forwards_per_chunk("self_forcing") == W.SELF_FORCING_FORWARDS
    sched = S.clip_schedule("unstep")
    cleans = [f for f in sched if f.clean]
    assert len(cleans) == 7 and all(f.label == 0.0 and f.sigma == 0.02 for f in cleans)
    first = [f for f in sched if f.chunk == 0 and not f.clean]
    assert [round(f.sigma, 4) for f in first] == [1.0, 0.9375, 0.8333, 0.625]
    later = [f for f in sched if f.chunk == 3 and not f.clean]
    assert [round(f.sigma, 4) for f in later] == [1.0, 0.8333]
    # each step hands the latent to the next step's level; the last one to the clean level
    assert first[-1].next_sigma == 0.02 and later[0].next_sigma == later[1].sigma


def test_renoise_oracle_closed_forms():
    g = torch.Generator().manual_seed(0)
    x = torch.randn(1000, generator=g).to(torch.bfloat16)
    e = torch.randn(1000, generator=g).to(torch.bfloat16)
    xb, eb = W.bits(x), W.bits(e)
    np.testing.assert_array_equal(oracle.renoise(xb, eb, 0.0), oracle.bf16_to_f64(xb))
    np.testing.assert_array_equal(oracle.renoise(xb, eb, 1.0), oracle.bf16_to_f64(eb))
    mid = oracle.renoise(xb, eb, 0.5)
    np.testing.assert_allclose(mid, 0.5 * (oracle.bf16_to_f64(xb) + oracle.bf16_to_f64(eb)),
                               rtol=0, atol=1e-15)
