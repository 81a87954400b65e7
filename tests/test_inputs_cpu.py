"""The seeded input generators (shared by the tests, bench and smoke), on CPU: determinism,
shapes and dtypes, and that the logit variant of the WKV-6 inputs is the same draw as the
decay variant."""
import numpy as np
import pytest
import torch

import oracle
from wkv_recurrence_02_b200 import inputs


def test_same_seed_same_draws():
    a = inputs.wkv6_inputs(2, 9, 3, 64, "bf16", seed=5, s0_std=0.1)
    b = inputs.wkv6_inputs(2, 9, 3, 64, "bf16", seed=5, s0_std=0.1)
    for n in a:
        assert torch.equal(a[n], b[n]), n
    c = inputs.wkv6_inputs(2, 9, 3, 64, "bf16", seed=6, s0_std=0.1)
    assert not torch.equal(a["r"], c["r"])


def test_shapes_and_dtypes():
    x = inputs.wkv6_inputs(2, 9, 3, 64, "bf16", seed=1, s0_std=0.1)
    for n in ("r", "k", "v", "w"):
        assert x[n].shape == (2, 9, 3, 64) and x[n].dtype == torch.bfloat16, n
    assert x["u"].shape == (3, 64) and x["u"].dtype == torch.float32
    assert x["s0"].shape == (2, 3, 64, 64) and x["s0"].dtype == torch.float32
    assert inputs.wkv6_inputs(1, 4, 2, 64, "fp32", seed=1)["s0"] is None
    y = inputs.wkv4_inputs(2, 5, 16, "bf16", seed=2)
    assert y["k"].shape == (2, 5, 16) and y["k"].dtype == torch.bfloat16
    assert y["w"].dtype == torch.float32 and bool((y["w"] > 0).all())
    g = inputs.norm_gate_inputs(2, 5, 3, 64, seed=3)
    assert g["g"].dtype == torch.bfloat16 and g["ln_w"].shape == (3, 64)


def test_logit_variant_is_the_same_draw():
    """decay="omega" returns omega_t in place of w_t from the same draws: r, k, v, u, s0 are
    identical, and the oracle's decay map of the fp32 logit gives the decay variant's w."""
    a = inputs.wkv6_inputs(2, 17, 3, 64, "fp32", seed=4, s0_std=0.1)
    b = inputs.wkv6_inputs(2, 17, 3, 64, "fp32", seed=4, s0_std=0.1, decay="omega")
    assert "w" not in b and "omega" not in a
    for n in ("r", "k", "v", "u", "s0"):
        assert torch.equal(a[n], b[n]), n
    w = oracle.decay_from_logit(b["omega"].double().numpy())
    np.testing.assert_allclose(w, a["w"].double().numpy(), rtol=1e-6, atol=0)
    assert float(a["w"].min()) > 0.0 and float(a["w"].max()) < 1.0


def test_bad_decay_option():
    with pytest.raises(ValueError):
        inputs.wkv6_inputs(1, 2, 1, 64, "fp32", seed=0, decay="log")
