"""The parity norms themselves (host only): the elementwise bar catches a localized
mistake that the per-head Frobenius bar lets through at full length."""
import numpy as np
import pytest

from parity import ELEM_TOL, TOL, check_parity, head_max_err, head_rel_err


def _head_block(T=4096, dv=128, noise=4e-3, seed=0):
    rng = np.random.default_rng(seed)
    ref = rng.standard_normal((1, T, 1, dv))
    got = ref + noise * rng.standard_normal(ref.shape)     # rounding-like error, spread out
    return got, ref


def test_rounding_noise_passes_both_bars():
    got, ref = _head_block()
    rel, mx = check_parity(got, ref, (0, 2), TOL["bf16"], "noise only")
    assert rel < 5e-3 and mx < ELEM_TOL["bf16"]


@pytest.mark.parametrize("mistake", ["zeroed", "from the previous token", "sign"])
def test_one_wrong_token_passes_frobenius_but_not_elementwise(mistake):
    """One token of 4096 wrong in all its 128 outputs: under the 2e-2 Frobenius bar
    (diluted by about 1/sqrt(4096)), far over the elementwise bar."""
    got, ref = _head_block()
    t = 2222
    if mistake == "zeroed":
        got[0, t] = 0.0
    elif mistake == "from the previous token":
        got[0, t] = ref[0, t - 1]
    else:
        got[0, t] = -ref[0, t]
    if mistake == "zeroed":
        assert head_rel_err(got, ref, (0, 2)) < TOL["bf16"]
    assert head_max_err(got, ref, (0, 2)) > 10 * ELEM_TOL["bf16"]
    with pytest.raises(AssertionError):
        check_parity(got, ref, (0, 2), TOL["bf16"], mistake)


def test_norms_are_per_head():
    """A head of small outputs is judged against its own RMS, not the batch's."""
    rng = np.random.default_rng(1)
    ref = rng.standard_normal((2, 64, 3, 16))
    ref[:, :, 1] *= 1e-3
    got = ref.copy()
    got[0, 5, 1, 3] += 1e-3 * 0.5          # half that head's RMS
    assert head_max_err(got, ref, (0, 2)) > 0.3
    assert head_rel_err(got, ref, (0, 2)) > 0.0
    assert head_max_err(ref, ref, (0, 2)) == 0.0
