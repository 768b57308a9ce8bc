"""The library's adaptive draft length (a host function of the C ABI) against the oracle:
the same k on random counts and costs (both sides decide in double, in the same order),
and argument validation."""
import numpy as np
import pytest

import sparse_dense_kv_b200 as s3r
from oracle import s3r_oracle as O


@pytest.mark.parametrize("seed", range(300))
def test_choose_horizon_matches_oracle(seed):
    rng = np.random.default_rng(seed)
    k_max = int(rng.integers(1, 9))
    dec = rng.integers(0, 200, size=k_max).astype(float)
    if seed % 3 == 0:
        dec = dec * rng.random(k_max)              # decayed (non-integer) counts
    acc = np.floor(dec * rng.random(k_max) ** (0.3 if seed % 2 else 3.0))
    c_d, c_v = float(rng.uniform(1, 100)), float(rng.uniform(1, 2000))
    pa, pw = float(rng.uniform(0, 1)), float(rng.choice([0.5, 4.0, 16.0]))
    want = O.choose_horizon(acc.tolist(), dec.tolist(), c_d, c_v, k_max, pa, pw)
    assert s3r.s3r_choose_horizon(acc.tolist(), dec.tolist(), c_d, c_v, pa, pw) == want


def test_choose_horizon_hand_worked_case():
    alpha = [0.66, 0.67, 0.64, 0.78, 1.0, 0.57]
    assert s3r.s3r_choose_horizon([a * 1e6 for a in alpha], [1e6] * 6, 57.0, 730.0, 0.5, 0.0) == 5


@pytest.mark.parametrize("args", [
    ([1.0] * 9, [1.0] * 9, 1.0, 1.0, 0.5, 1.0),      # k_max > 8
    ([1.0], [1.0], 0.0, 1.0, 0.5, 1.0),              # c_draft <= 0
    ([1.0], [1.0], 1.0, float("inf"), 0.5, 1.0),     # c_verify not finite
    ([1.0], [1.0], 1.0, 1.0, 1.5, 1.0),              # prior outside [0, 1]
    ([1.0], [1.0], 1.0, 1.0, 0.5, -1.0),             # negative prior weight
    ([-1.0], [1.0], 1.0, 1.0, 0.5, 1.0),             # negative count
    ([0.0], [0.0], 1.0, 1.0, 0.5, 0.0),              # a position with no evidence and no prior
])
def test_choose_horizon_rejects_bad_arguments(args):
    with pytest.raises(s3r.S3RError):
        s3r.s3r_choose_horizon(*args)
