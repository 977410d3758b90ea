"""Shared helpers of the GPU parity tests: tolerances and comparisons.

Tolerances (bf16 inputs, fp32 accumulation): output O max-abs <= 1e-2 and
relative RMS <= 5e-3; LSE max-abs <= 1e-3; cached states written this step
the same; plans, counts and untouched cache slots bit-exact.
"""

import numpy as np

O_MAX_ABS = 1e-2
O_REL_RMS = 5e-3
L_MAX_ABS = 1e-3


def to_np(t):
    return t.detach().float().cpu().numpy().astype(np.float64)


def rel_rms(a, b):
    den = np.sqrt(np.mean(b * b))
    return float(np.sqrt(np.mean((a - b) ** 2)) / den) if den > 0 else float(np.sqrt(np.mean(a * a)))


BF16_QUANTUM = 2.0 ** -8     # relative spacing of bf16 values at the bottom of a binade


def check_out(o_gpu, o_ref, what="O", max_abs=O_MAX_ABS, rel=O_REL_RMS, output_scaled=False):
    """max-abs and relative-RMS check.  ``output_scaled`` (unit-variance
    stress inputs only, where |O| reaches 4 and a bf16 output's own rounding
    exceeds 1e-2) widens the max-abs bound by one bf16 quantum of |O_ref|."""
    o_gpu = np.asarray(o_gpu, dtype=np.float64)
    assert np.all(np.isfinite(o_gpu)), f"{what}: non-finite values"
    err = np.abs(o_gpu - o_ref)
    bound = max_abs + (BF16_QUANTUM * np.abs(o_ref) if output_scaled else 0.0)
    ma, rr = float(err.max()), rel_rms(o_gpu, o_ref)
    assert np.all(err <= bound), f"{what}: max-abs {ma:.3e} > {max_abs} (+bf16 quantum: {output_scaled})"
    assert rr <= rel, f"{what}: rel-RMS {rr:.3e} > {rel}"
    return ma, rr


def check_lse(l_gpu, l_ref, what="LSE", max_abs=L_MAX_ABS):
    l_gpu = np.asarray(l_gpu, dtype=np.float64)
    neg = ~np.isfinite(l_ref)
    assert np.array_equal(~np.isfinite(l_gpu), neg), f"{what}: -inf pattern differs"
    if (~neg).any():
        ma = float(np.abs(l_gpu[~neg] - l_ref[~neg]).max())
        assert ma <= max_abs, f"{what}: max-abs {ma:.3e} > {max_abs}"
        return ma
    return 0.0
