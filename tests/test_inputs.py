"""The seeded input generator: deterministic, right shapes, right value ranges."""
import torch

from gated_delta_rule_100_b200 import inputs


def test_prefill_is_deterministic_and_in_range():
    a = inputs.make_prefill(2, 70, 3, 64, 32, decay=0.1, h0_std=0.02, seed=5)
    b = inputs.make_prefill(2, 70, 3, 64, 32, decay=0.1, h0_std=0.02, seed=5)
    for key in a:
        assert torch.equal(a[key], b[key]), key
    assert a["q"].dtype == torch.bfloat16 and a["q"].shape == (2, 70, 3, 64)
    assert a["v"].shape == (2, 70, 3, 32) and a["beta"].shape == (2, 70, 3)
    assert a["h0"].shape == (2, 3, 64, 32)
    assert (a["g"] <= 0).all() and (a["g"] > -5).all()
    assert ((a["beta"] > 0) & (a["beta"] < 1)).all()
    n = a["k"].float().norm(dim=-1)
    assert torch.allclose(n, torch.ones_like(n), atol=1e-2)


def test_seed_changes_values():
    a = inputs.make_prefill(1, 16, 1, 64, 64, decay=0.1, seed=0)
    b = inputs.make_prefill(1, 16, 1, 64, 64, decay=0.1, seed=1)
    assert not torch.equal(a["q"], b["q"])
    assert a["h0"] is None


def test_decode_shapes():
    d = inputs.make_decode(4, 2, 64, 64, decay=0.05, state_std=0.02, steps=3, seed=0)
    assert d["state"].shape == (4, 2, 64, 64)
    assert d["q"].shape == (3, 4, 2, 64) and d["beta"].shape == (3, 4, 2)


def test_digest_stable():
    a = inputs.make_prefill(1, 8, 1, 64, 64, decay=0.1, seed=0)
    assert inputs.digest(a["q"], a["g"]) == inputs.digest(a["q"], a["g"])
