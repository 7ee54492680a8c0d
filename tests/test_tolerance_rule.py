"""The output tolerance adds half a bf16 ulp of the exact value: check that
term against actual round-to-nearest bf16 conversion (no GPU)."""
import numpy as np

import moe_harness as MH
from sigmoid_routed_mixture_b200 import workloads as W


def test_half_ulp_bounds_bf16_rounding_tightly():
    rng = np.random.default_rng(0)
    v = np.concatenate([rng.standard_normal(200000) * s for s in (0.01, 1.0, 3.0, 40.0)])
    v = v.astype(np.float32).astype(np.float64)  # one rounding only: fp32 -> bf16
    r = W.bf16_bits_to_f32(W.f32_to_bf16_bits(v.astype(np.float32))).astype(np.float64)
    hu = MH.half_ulp_bf16(v)
    err = np.abs(r - v)
    assert np.all(err <= hu * (1 + 1e-6) + 1e-30)
    assert np.max(err / hu) > 0.99  # the bound is attained, not loose


def test_within_tolerance_rule():
    y_o = np.array([20.0 + 0.0624, 1.0, -1.0])
    rms = np.sqrt(np.mean(y_o ** 2))
    ok, rel, _ = MH.within_tolerance(np.array([20.0, 1.0, -1.0]), y_o)
    assert ok and rel > 0.0624 / rms * 0.99
    ok, _, _ = MH.within_tolerance(np.array([20.0, 1.0 + 0.03 * rms, -1.0]), y_o)
    assert not ok
