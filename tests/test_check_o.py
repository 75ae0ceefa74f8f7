"""CPU checks of the O comparison helper: where a 16-bit output cannot be
within 1e-2 of the oracle, the element is compared with the oracle rounded
to that dtype, and every such element is recorded (never dropped silently)."""
import numpy as np
import pytest
import torch

import helpers


def test_rounded_comparison_is_recorded():
    # 5 + 2^-6: bf16 has an ulp of 2^-5 at 5, so the nearest bf16 value is
    # 2^-6 = 0.0156 away, more than the 1e-2 bound
    ref = np.full((1, 4096), 0.5)  # mean-abs stays below 1e-3 over the many exact elements
    ref[0, 7] = 5.0 + 2.0 ** -6
    gpu = torch.from_numpy(ref).to(torch.bfloat16)
    n0 = len(helpers.ROUNDED_COMPARISONS)
    raw, _ = helpers.check_o(gpu, ref, "bf16 at |O| = 5")
    assert raw == pytest.approx(2.0 ** -6)
    recs = helpers.ROUNDED_COMPARISONS[n0:]
    assert len(recs) == 1 and recs[0]["elements"] == 1
    assert recs[0]["raw_max"] == pytest.approx(2.0 ** -6) and recs[0]["err_vs_rounded_max"] == 0.0


def test_rounded_comparison_still_fails_one_ulp_off():
    ref = np.full((1, 4096), 0.5)
    ref[0, 0] = 5.0 + 2.0 ** -6
    rounded = torch.from_numpy(ref).to(torch.bfloat16).double().numpy()
    gpu = torch.from_numpy(rounded + 2.0 ** -5).to(torch.bfloat16)  # one bf16 ulp beyond the rounding
    with pytest.raises(AssertionError, match="held against the oracle rounded"):
        helpers.check_o(gpu, ref, "one ulp off")


def test_representable_elements_use_the_raw_bound():
    ref = np.ones((1, 4096))
    ref[0, 5] = 1.0 + 2.0 ** -9  # bf16 rounding error 2^-9 < 1e-2: the raw bound applies
    n0 = len(helpers.ROUNDED_COMPARISONS)
    helpers.check_o(torch.from_numpy(ref).to(torch.bfloat16), ref, "small")
    assert len(helpers.ROUNDED_COMPARISONS) == n0
    with pytest.raises(AssertionError):
        off = ref.copy()
        off[0, 3] += 0.02
        helpers.check_o(torch.from_numpy(off).to(torch.bfloat16), ref, "small, off")
