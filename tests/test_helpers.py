"""The GPU tests' own helpers, checked on the CPU: the Gram-eigenvalue route to singular
values against LAPACK's SVD, and the update bound accepting the exactly rounded update and
rejecting one that is two ulps off."""
import numpy as np
import pytest

import oracle as orc
from gpu_helpers import assert_update_within_bound, sv, sv_gram


@pytest.mark.parametrize("shape", [(40, 96), (96, 40), (64, 64)])
def test_sv_gram_matches_svd(shape):
    r = np.random.default_rng(5)
    x = r.standard_normal(shape)
    x /= np.linalg.norm(x, 2)           # sigma_max = 1, like a Newton-Schulz output
    assert np.max(np.abs(sv_gram(x) - sv(x))) <= 1e-12


def test_update_bound_accepts_exact_rounding_and_rejects_two_ulps():
    r = np.random.default_rng(6)
    W0 = orc.round_to_bf16(r.standard_normal((32, 48)) * 0.02)
    O = orc.round_to_bf16(r.standard_normal((32, 48)) * 0.05)
    lr, wd, s = 0.02, 0.1, 1.3
    W1 = orc.round_to_bf16(orc.muon_update(W0, O, lr, wd, s))
    assert_update_within_bound(W1, W0, O, lr, wd, s, bf16=True)
    bad = W1.copy()
    bad[3, 7] = orc.round_to_bf16(bad[3, 7] * (1 + 2.0 ** -6))   # about two bf16 ulps away
    with pytest.raises(AssertionError):
        assert_update_within_bound(bad, W0, O, lr, wd, s, bf16=True)
