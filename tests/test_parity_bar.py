"""CPU checks of the GPU parity bar itself (no GPU needed).

* Every input named in DERIVED_BAR really puts the flat 5e-3 bar out of reach of the method: the
  correctly rounded bf16 value of the exact result on the bf16-folded W* already misses it, so no
  kernel that rounds its output once could meet it there.
* check_bf16 accepts that correctly rounded value and rejects a result one bf16 ulp off at the largest
  output, and a result that misses the flat bar while inside the half-ulp band (a wrong reference).
"""

import numpy as np
import pytest

import flashnorm_inputs as I
from oracle import flashnorm_oracle as O
from tests.test_gpu_parity import BF16_TOL, DERIVED_BAR, check_bf16


def _rounded(v):
    return O.bf16_to_f64(O.f64_to_bf16(v))


@pytest.mark.parametrize("case", sorted(DERIVED_BAR), ids=str)
def test_derived_bar_cases_miss_the_flat_bar_when_rounded_correctly(case):
    kind, M, d, N, seed = case
    bits = I.Workload("t", kind, M, d, N, 1e-5, seed=seed).draw()
    ref = O.reference_output(kind, bits, 1e-5)
    ex = O.exact_operand_output(kind, bits, O.fold_bf16(bits["w"], bits["g"]), 1e-5)
    assert O.rel_err(_rounded(ex), ref) > BF16_TOL
    check_bf16(_rounded(ex), ref, ex, derived=True)


def test_check_bf16_accepts_correct_rounding_and_rejects_an_ulp_off():
    bits = I.Workload("t", "linear", 24, 576, 96, 1e-5, seed=3).draw()
    ref = O.reference_output("linear", bits, 1e-5)
    ex = O.exact_operand_output("linear", bits, O.fold_bf16(bits["w"], bits["g"]), 1e-5)
    y = _rounded(ex)
    assert check_bf16(y, ref, ex) <= BF16_TOL
    i = np.unravel_index(np.argmax(np.abs(ex)), ex.shape)
    bad = y.copy()
    _, e = np.frexp(bad[i])
    bad[i] += np.sign(ex[i]) * np.ldexp(1.0, e - 8)  # one ulp away from the exact value
    with pytest.raises(AssertionError):
        check_bf16(bad, ref, ex)
    # a reference that is off by 1% (a wrong definition) fails the flat bar
    with pytest.raises(AssertionError):
        check_bf16(y, ref * 1.01, ex)
