"""Pins of the oracle's router.

"DeepSeek-V3 Technischer Bericht", Methode section 2: s_{i,t} =
Sigmoid(u_t^T e_i); expert i is selected when s_{i,t} + b_i is among the K_r
largest of {s_{j,t} + b_j}; g'_{i,t} = s_{i,t} on selected experts and 0
elsewhere; g is g' normalised.  Pins: sigmoid affinities against a library
sigmoid of a library matmul, top-K_r against brute force over every K_r-subset,
gates summing to one, invariance to a common bias shift, K_r = N_r selecting
every expert, and group-limited routing against brute force over group
subsets (that rule is this build's reading; the pages do not state it).
"""
import itertools

import numpy as np
import pytest
from scipy.special import expit

from moe_synth import TINY, gen_bias, gen_router, gen_x, gen_mixture_x


def _tiny(seed=0):
    x = gen_x(64, TINY["H"], seed)
    Wr = gen_router(TINY["Nr"], TINY["H"], seed)
    b = gen_bias(TINY["Nr"], seed)
    return x, Wr, b


def test_affinity_is_sigmoid_of_logits(oracle_lib):
    x, Wr, b = _tiny()
    cf = oracle_lib.cfg(TINY["H"], TINY["I"], TINY["Nr"], TINY["Kr"])
    idx, gate, gap, s = oracle_lib.route(cf, x, Wr, b, want_s=True)
    z = x.double().numpy() @ Wr.double().numpy().T
    assert np.allclose(s, expit(z), rtol=1e-13, atol=0)


def test_topk_brute_force_and_gates(oracle_lib):
    x, Wr, b = _tiny(1)
    Nr, Kr = TINY["Nr"], TINY["Kr"]
    cf = oracle_lib.cfg(TINY["H"], TINY["I"], Nr, Kr)
    idx, gate, gap, s = oracle_lib.route(cf, x, Wr, b, want_s=True)
    bf = b.numpy().astype(np.float32)
    subsets = np.array(list(itertools.combinations(range(Nr), Kr)))
    assert len(subsets) == 1820
    for t in range(x.shape[0]):
        c = s[t].astype(np.float32) + bf          # the decision value, FP32
        sums = c.astype(np.float64)[subsets].sum(axis=1)
        best = subsets[np.argmax(sums)]
        assert set(idx[t].tolist()) == set(best.tolist()), t
        # idx in descending-score order
        assert np.all(np.diff(c[idx[t]]) <= 0)
        assert abs(gate[t].sum() - 1.0) < 1e-12
        assert np.allclose(gate[t], s[t, idx[t]] / s[t, idx[t]].sum(), rtol=1e-14)
        rest = np.setdiff1d(np.arange(Nr), idx[t])
        assert gap[t] == pytest.approx(float(c[idx[t]].min() - c[rest].max()), abs=0)


def test_bias_only_selects(oracle_lib):
    # A large bias on one expert forces its selection, but its gate stays
    # proportional to its unbiased affinity s.
    x, Wr, b = _tiny(2)
    Nr, Kr = TINY["Nr"], TINY["Kr"]
    cf = oracle_lib.cfg(TINY["H"], TINY["I"], Nr, Kr)
    b2 = b.clone()
    b2[3] = 10.0
    idx, gate, gap, s = oracle_lib.route(cf, x, Wr, b2, want_s=True)
    assert np.all((idx == 3).sum(axis=1) == 1)
    for t in range(x.shape[0]):
        assert np.allclose(gate[t], s[t, idx[t]] / s[t, idx[t]].sum(), rtol=1e-14)


def test_common_bias_shift_changes_nothing(oracle_lib):
    x, Wr, b = _tiny(3)
    cf = oracle_lib.cfg(TINY["H"], TINY["I"], TINY["Nr"], TINY["Kr"])
    i0, g0, gap0, _ = oracle_lib.route(cf, x, Wr, b)
    i1, g1, gap1, _ = oracle_lib.route(cf, x, Wr, b + 0.25)
    clear = gap0 > 1e-5
    assert clear.mean() > 0.9
    for t in np.nonzero(clear)[0]:
        assert set(i0[t]) == set(i1[t])
    assert np.allclose(g0[clear], g1[clear], rtol=1e-14)


def test_all_experts_when_k_equals_n(oracle_lib):
    x, Wr, b = _tiny(4)
    Nr = TINY["Nr"]
    cf = oracle_lib.cfg(TINY["H"], TINY["I"], Nr, Nr)
    idx, gate, gap, s = oracle_lib.route(cf, x, Wr, b, want_s=True)
    for t in range(x.shape[0]):
        assert sorted(idx[t].tolist()) == list(range(Nr))
        assert np.allclose(np.sort(gate[t]), np.sort(s[t] / s[t].sum()), rtol=1e-13)


def test_group_limited_brute_force(oracle_lib):
    H, Nr, Kr, G, TG = 256, 16, 4, 4, 2
    x, _ = gen_mixture_x(96, H, 5, n_centroids=4)
    Wr = gen_router(Nr, H, 5)
    b = gen_bias(Nr, 5)
    cf = oracle_lib.cfg(H, 128, Nr, Kr, 1, G, TG)
    idx, gate, gap, s = oracle_lib.route(cf, x, Wr, b, want_s=True)
    bf = b.numpy().astype(np.float32)
    gs = Nr // G
    for t in range(x.shape[0]):
        c = s[t].astype(np.float32) + bf
        score = np.array([np.float32(np.sort(c[g * gs:(g + 1) * gs])[-1]) + np.float32(np.sort(c[g * gs:(g + 1) * gs])[-2])
                          for g in range(G)], dtype=np.float32)
        gsets = list(itertools.combinations(range(G), TG))
        best_groups = max(gsets, key=lambda S: (sum(float(score[g]) for g in S), [-g for g in S]))
        allowed = [j for j in range(Nr) if j // gs in best_groups]
        esets = list(itertools.combinations(allowed, Kr))
        best = max(esets, key=lambda S: sum(float(c[j]) for j in S))
        if gap[t] > 1e-6:
            assert set(idx[t].tolist()) == set(best), t
        assert all(j // gs in best_groups for j in idx[t]) or gap[t] <= 1e-6
        assert abs(gate[t].sum() - 1.0) < 1e-12
