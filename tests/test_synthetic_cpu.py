"""The seeded input recipe (the input distributions the parity tests and the
benchmark use) holds the properties it is documented to have."""
import dataclasses

import numpy as np

from oracle import formats as F
from routed_nvfp4_expert_b200 import synthetic as syn


def test_nvfp4_bank_dequantises_to_the_target_std():
    for sigma in (0.02, 0.0064):
        c, s, t = syn.nvfp4_bank(0, "gate", 4, 128, 512, sigma)
        w = np.stack([F.nvfp4_dequant(c[e], s[e], t[e]) for e in range(4)])
        assert abs(w.std() / sigma - 1.0) < 0.08, w.std()
        assert abs(w.mean()) < 0.02 * sigma


def test_nvfp4_bank_scale_exponents_and_determinism():
    c, s, t = syn.nvfp4_bank(0, "up", 2, 64, 256, 0.02)
    exp_field = (s >> 3) & 0xF
    frac = [np.mean(exp_field == v) for v in (12, 13, 14)]
    assert np.all(np.isin(exp_field, (12, 13, 14)))
    assert abs(frac[0] - 0.25) < 0.03 and abs(frac[1] - 0.5) < 0.03 and abs(frac[2] - 0.25) < 0.03
    c2, s2, t2 = syn.nvfp4_bank(0, "up", 2, 64, 256, 0.02)
    assert np.array_equal(c, c2) and np.array_equal(s, s2) and np.array_equal(t, t2)   # seeded
    c3, _, _ = syn.nvfp4_bank(1, "up", 2, 64, 256, 0.02)
    assert not np.array_equal(c, c3)


def test_router_and_x_distributions():
    wl = dataclasses.replace(syn.WORKLOADS["decode_t1"], T=256)
    d = syn.make_router_and_x(wl, seed=0)
    x = F.bf16_value(d["x"])
    assert abs(x.std() - 1.0) < 0.02
    assert abs(d["router_w"].std() * np.sqrt(wl.H) - 1.0) < 0.02
    assert abs(d["router_bias"].std() - 0.5) < 0.1


def test_stress_recipe_exact_values():
    wl = dataclasses.replace(syn.WORKLOADS["stress_t16384"], T=1000)
    d = syn.make_router_and_x(wl, seed=0)
    S, j, tie = d["skew_set"], d["tie_column"], d["tie_tokens"]
    assert len(S) == 16 and len(tie) == 10
    assert np.all(d["router_bias"][S] == np.float32(3.0))
    assert np.all(d["router_w"][S, j] == 0.0)
    x = F.bf16_value(d["x"])
    assert np.all(x[tie, j] == 8.0) and np.count_nonzero(x[tie]) == len(tie)
    others = np.setdiff1d(np.arange(wl.T), tie)
    assert abs(x[others].std() / wl.x_scale - 1.0) < 0.02      # activations scaled by x_scale
