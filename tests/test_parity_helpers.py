"""The comparison helpers of the GPU parity tests, checked on the CPU.

The output bar must catch an epilogue mistake confined to one column of the
output (a wrong column index, a dropped store, a swapped vector lane), which
the per-token L2 error alone lets through at d = 4096. The mistakes are
planted in copies of an oracle result, never in the library.
"""

import numpy as np
import pytest

from parity_util import TOL_BF16, TOL_F32, assert_rows_close, elem_rel_err, token_rel_err


def _bf16_round(a):
    """Round float64 values to the nearest bf16 (ties to even), as float64."""
    f = np.asarray(a, dtype=np.float32)
    u = f.view(np.uint32).astype(np.uint64)
    u = (u + 0x7FFF + ((u >> 16) & 1)) & 0xFFFF0000
    return u.astype(np.uint32).view(np.float32).astype(np.float64)


def _reference(T=64, d=4096, seed=0):
    rng = np.random.default_rng(seed)
    return rng.standard_normal((T, d)) * rng.uniform(0.1, 3.0, (T, 1))


def test_bf16_rounding_passes():
    ref = _reference()
    y = _bf16_round(ref)
    rel, elem, glob = assert_rows_close(y, ref, TOL_BF16)
    assert rel < 2 ** -8 and elem < 2 ** -8


@pytest.mark.parametrize("slip", ["zero", "neighbour", "negated", "half"])
def test_single_column_slip_fails_the_element_bar(slip):
    ref = _reference()
    y = _bf16_round(ref)
    c = 1234
    if slip == "zero":
        y[:, c] = 0.0
    elif slip == "neighbour":
        y[:, c] = y[:, c + 1]
    elif slip == "negated":
        y[:, c] = -y[:, c]
    else:
        y[:, c] *= 0.5
    # the per-token L2 bar passes most tokens of this output (it fails only
    # those whose slipped element happens to be large) ...
    # (a negated column doubles the error and sits at the bar)
    per_token = [token_rel_err(y[t:t + 1], ref[t:t + 1])[0] for t in range(ref.shape[0])]
    assert np.median(per_token) < (2 if slip == "negated" else 1) * TOL_BF16
    # ... the element bar fails it
    elem, _ = elem_rel_err(y, ref)
    assert elem > TOL_BF16
    with pytest.raises(AssertionError):
        assert_rows_close(y, ref, TOL_BF16)


def test_one_wrong_element_of_one_token_fails():
    ref = _reference()
    y = _bf16_round(ref)
    t, i = 17, 4000
    y[t, i] += 0.05 * np.abs(ref[t]).max()
    with pytest.raises(AssertionError):
        assert_rows_close(y, ref, TOL_BF16)


def test_fp32_bar():
    ref = _reference(T=32, d=128, seed=3)
    y = ref.astype(np.float32).astype(np.float64)
    assert_rows_close(y, ref, TOL_F32)
    y[5, 7] += 2e-5 * np.abs(ref[5]).max()
    with pytest.raises(AssertionError):
        assert_rows_close(y, ref, TOL_F32)


def test_zero_rows_must_be_exact():
    ref = _reference(T=8, d=64)
    ref[3] = 0.0
    y = ref.copy()
    assert_rows_close(y, ref, TOL_BF16)
    y[3, 10] = 1e-30
    with pytest.raises(AssertionError):
        assert_rows_close(y, ref, TOL_BF16)
