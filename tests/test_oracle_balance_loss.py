"""Pins of the oracle's sequence-wise balance loss.

"DeepSeek-V3 Technischer Bericht", Methode section 2, names the loss and its
weight alpha = 0.0001; the form checked here is the technical report's
(loss = alpha * sum_i f_i P_i with f_i = N_r / (K_r L) * picks_i and P_i the
sequence mean of the normalised affinities).  The pins are closed forms of
that definition: each fails if a factor, the normalisation or an axis is
wrong.
"""
import numpy as np
import pytest

ALPHA = 1e-4


def _random_idx(rng, T, Nr, Kr):
    return np.stack([rng.choice(Nr, Kr, replace=False) for _ in range(T)]).astype(np.int32)


def test_hand_worked_two_expert_case(oracle_lib):
    # Nr = 2, Kr = 1, L = 2; both tokens pick expert 0.
    # f = [2/(1*2) * 2, 0] = [2, 0]; P_0 = (3/4 + 1/2) / 2 = 5/8 -> loss = 2 * 5/8 * alpha
    s = np.array([[3.0, 1.0], [1.0, 1.0]])
    idx = np.array([[0], [0]])
    assert oracle_lib.seq_balance_loss(s, idx, 2, 1, 2, ALPHA)[0] == pytest.approx(1.25 * ALPHA, rel=1e-15)


@pytest.mark.parametrize("Nr,Kr,L", [(16, 4, 64), (256, 8, 256), (8, 8, 4)])
def test_equal_affinities_give_alpha_for_any_selection(oracle_lib, Nr, Kr, L):
    # P_i = 1/N_r for every i and sum_i f_i = N_r, so the loss is alpha
    rng = np.random.default_rng(Nr + Kr + L)
    s = np.full((L, Nr), 0.37)
    idx = _random_idx(rng, L, Nr, Kr)
    assert oracle_lib.seq_balance_loss(s, idx, Nr, Kr, L, ALPHA)[0] == pytest.approx(ALPHA, rel=1e-12)


@pytest.mark.parametrize("Nr,Kr", [(16, 4), (256, 8), (6, 2)])
def test_balanced_selection_gives_alpha_for_any_affinities(oracle_lib, Nr, Kr):
    # every expert picked equally often: f_i = 1, and sum_i P_i = 1
    rng = np.random.default_rng(Nr * Kr)
    L = Nr  # token t picks experts t, t+1, ..., t+Kr-1 (mod Nr): each expert Kr times
    idx = np.array([[(t + k) % Nr for k in range(Kr)] for t in range(L)])
    s = rng.uniform(0.01, 1.0, size=(L, Nr))
    assert oracle_lib.seq_balance_loss(s, idx, Nr, Kr, L, ALPHA)[0] == pytest.approx(ALPHA, rel=1e-12)


@pytest.mark.parametrize("Nr,Kr,L", [(16, 4, 32), (256, 8, 64)])
def test_fully_collapsed_routing_gives_alpha_nr_over_kr(oracle_lib, Nr, Kr, L):
    # every token picks experts 0..Kr-1 and puts all its affinity on them,
    # evenly: f_i = N_r / K_r and P_i = 1 / K_r there, 0 elsewhere
    s = np.zeros((L, Nr))
    s[:, :Kr] = 0.8
    idx = np.tile(np.arange(Kr), (L, 1))
    assert oracle_lib.seq_balance_loss(s, idx, Nr, Kr, L, ALPHA)[0] == pytest.approx(ALPHA * Nr / Kr, rel=1e-12)


def test_per_token_scaling_of_affinities_changes_nothing(oracle_lib):
    rng = np.random.default_rng(5)
    Nr, Kr, L = 16, 4, 48
    s = rng.uniform(0.05, 0.95, size=(L, Nr))
    idx = _random_idx(rng, L, Nr, Kr)
    a = oracle_lib.seq_balance_loss(s, idx, Nr, Kr, L, ALPHA)
    b = oracle_lib.seq_balance_loss(s * rng.uniform(0.5, 4.0, size=(L, 1)), idx, Nr, Kr, L, ALPHA)
    np.testing.assert_allclose(a, b, rtol=1e-13)


def test_sequences_are_independent_and_alpha_is_a_factor(oracle_lib):
    rng = np.random.default_rng(6)
    Nr, Kr, L = 16, 4, 32
    s = rng.uniform(0.05, 0.95, size=(3 * L, Nr))
    idx = _random_idx(rng, 3 * L, Nr, Kr)
    whole = oracle_lib.seq_balance_loss(s, idx, Nr, Kr, L, ALPHA)
    parts = [oracle_lib.seq_balance_loss(s[q * L:(q + 1) * L], idx[q * L:(q + 1) * L], Nr, Kr, L, ALPHA)[0]
             for q in range(3)]
    assert whole.shape == (3,) and np.array_equal(whole, np.array(parts))
    np.testing.assert_allclose(oracle_lib.seq_balance_loss(s, idx, Nr, Kr, L, 1.0) * ALPHA, whole, rtol=1e-15)
    # a skewed selection costs more than the balanced floor
    assert (whole > 0).all()
