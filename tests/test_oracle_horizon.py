"""Pins for the oracle's adaptive draft length: the geometric closed form of the expected
tokens for a flat acceptance, the limits alpha = 1 and alpha = 0, a hand-worked case, and
the prior for positions never decided."""
import numpy as np
import pytest

from oracle import s3r_oracle as O


def geometric_best(alpha, c_d, c_v, k_max):
    """argmax_k (1 - alpha^(k+1)) / (1 - alpha) / (k c_d + c_v), smallest k on ties."""
    rates = [((k + 1) if alpha == 1.0 else (1 - alpha ** (k + 1)) / (1 - alpha)) / (k * c_d + c_v)
             for k in range(1, k_max + 1)]
    return int(np.argmax(rates)) + 1


@pytest.mark.parametrize("alpha", [0.05, 0.3, 0.6, 0.8, 0.9, 0.97])
@pytest.mark.parametrize("c_d,c_v", [(57.0, 730.0), (1.0, 1.0), (40.0, 28.0), (5.0, 300.0)])
def test_flat_acceptance_matches_the_geometric_closed_form(alpha, c_d, c_v):
    # counts that give exactly alpha at every position, no prior
    dec = [1000.0] * 8
    acc = [alpha * 1000.0] * 8
    assert O.choose_horizon(acc, dec, c_d, c_v, 8, prior_weight=0.0) == geometric_best(alpha, c_d, c_v, 8)


def test_limits():
    ones, zeros, dec = [50.0] * 8, [0.0] * 8, [50.0] * 8
    # every draft accepted: (k + 1) / (k c_d + c_v) grows with k when c_v > c_d
    assert O.choose_horizon(ones, dec, 10.0, 100.0, 8, prior_weight=0.0) == 8
    assert O.choose_horizon(ones, dec, 100.0, 10.0, 8, prior_weight=0.0) == 1
    # nothing accepted: one token per round whatever k, so the cheapest round
    assert O.choose_horizon(zeros, dec, 10.0, 100.0, 8, prior_weight=0.0) == 1


def test_hand_worked_case():
    # acceptance by position as measured on the 32-request Qwen3-8B-shaped workload,
    # draft step 57 us, verify + selection + sampling 730 us:
    # k:     1      2       3        4          5          6
    # tau:  1.66  2.1022  2.385208  2.60595424 2.82670048 2.9525258368
    # cost: 787   844     901       958        1015       1072
    # rate: .0021093 .0024908 .0026473 .0027202 .0027849 .0027542 -> k = 5
    alpha = [0.66, 0.67, 0.64, 0.78, 1.0, 0.57]
    dec = [1e6] * 6
    acc = [a * 1e6 for a in alpha]
    assert O.choose_horizon(acc, dec, 57.0, 730.0, 6, prior_weight=0.0) == 5


def test_prior_fills_undecided_positions():
    # positions 7 and 8 never decided: their acceptance is the prior
    acc = [90.0] * 6 + [0.0, 0.0]
    dec = [100.0] * 6 + [0.0, 0.0]
    est = O.acceptance_estimate(acc, dec, 0.5, 4.0)
    assert est[6] == est[7] == 0.5
    assert abs(est[0] - (90 + 2) / 104) < 1e-15
    # with a pessimistic prior the extra positions are not worth drafting
    assert O.choose_horizon(acc, dec, 57.0, 730.0, 8, prior_alpha=0.0, prior_weight=4.0) <= 6


def test_decayed_counts_and_pooled_prior_hand_worked():
    # decay 1/2: accepted (4, 2) -> (4/2 + 2, 2/2 + 0) = (4, 1); decided (8, 8) -> (6, 6)
    acc, dec, prior, k = O.horizon_step([4.0, 2.0], [8.0, 8.0], [2, 0], [2, 2], 0.5, 1.0, 4.0, 2,
                                        prior_alpha=None, prior_weight=4.0)
    assert acc == [4.0, 1.0] and dec == [6.0, 6.0]
    assert prior == 5.0 / 12.0                      # (4 + 1) / (6 + 6)
    # alpha = ((4 + 4 * 5/12) / 10, (1 + 4 * 5/12) / 10) = (17/30, 8/30)
    # c_draft 1, c_verify 4: k=1 (47/30)/5 = .31333 > k=2 (1546/900)/6 = .28630
    assert k == 1
    # c_verify 40: k=1 (47/30)/41 = .038211 < k=2 (1546/900)/42 = .040899
    assert O.horizon_step([4.0, 2.0], [8.0, 8.0], [2, 0], [2, 2], 0.5, 1.0, 40.0, 2)[3] == 2
    # a fixed prior replaces the pooled one; decay 1 keeps every count
    acc, dec, prior, _ = O.horizon_step([4.0, 2.0], [8.0, 8.0], [2, 0], [2, 2], 1.0, 1.0, 4.0, 2,
                                        prior_alpha=0.25)
    assert acc == [6.0, 2.0] and dec == [10.0, 10.0] and prior == 0.25
    # nothing decided yet: the pooled prior is one half
    assert O.pooled_prior([0.0] * 4, [0.0] * 4, 4) == 0.5
