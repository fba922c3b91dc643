"""Pins of the oracle's integer grouping step: the per-expert histogram and the
expert-contiguous order of the (token, slot) assignments.

"DeepSeek-V3 Technischer Bericht" (xyznot.com/de), Methode section 2: each
routed expert i sees exactly the tokens whose top-K_r selection contains i.
The layer groups those (token, slot) pairs by expert; the order inside one
expert's run is this implementation's stable reading (token ascending, then
slot k), so that rows compare bit for bit.  The pins below fix the functions
against hand-worked values and against a brute-force definition written
without sorting primitives.
"""
import numpy as np
import pytest


def brute_order(idx, Nr):
    """Plain loops: for each expert in turn, walk the tokens in order and
    their slots in order, appending every slot that names the expert."""
    T, Kr = idx.shape
    order, offsets = [], [0]
    for e in range(Nr):
        for t in range(T):
            for k in range(Kr):
                if idx[t, k] == e:
                    order.append(t * Kr + k)
        offsets.append(len(order))
    return np.array(offsets), np.array(order)


def test_hand_worked_order(oracle_lib):
    # 4 tokens, 3 slots, 5 experts.  Expert 0 is picked by every token,
    # expert 3 by none; token 2 lists expert 4 before expert 0, so expert 0's
    # run must still follow token order (t2 after t1), and expert 4's run
    # takes t0 slot 2 before t2 slot 0 (token before slot).
    idx = np.array([[0, 1, 4],
                    [2, 0, 1],
                    [4, 0, 2],
                    [1, 2, 0]], np.int32)
    offsets, order = oracle_lib.expert_order(idx, 5)
    # expert 0: (t0,k0)=0 (t1,k1)=4 (t2,k1)=7 (t3,k2)=11
    # expert 1: (t0,k1)=1 (t1,k2)=5 (t3,k0)=9
    # expert 2: (t1,k0)=3 (t2,k2)=8 (t3,k1)=10
    # expert 3: none
    # expert 4: (t0,k2)=2 (t2,k0)=6
    assert offsets.tolist() == [0, 4, 7, 10, 10, 12]
    assert order.tolist() == [0, 4, 7, 11, 1, 5, 9, 3, 8, 10, 2, 6]
    assert oracle_lib.histogram(idx, 5).tolist() == [4, 3, 3, 0, 2]


def test_every_token_same_expert(oracle_lib):
    # one expert taken by every token (slot 0), the rest spread
    T, Kr, Nr = 7, 2, 4
    idx = np.array([[2, t % 2] for t in range(T)], np.int32)
    offsets, order = oracle_lib.expert_order(idx, Nr)
    assert offsets.tolist() == [0, 4, 7, 14, 14]
    assert order[7:14].tolist() == [t * Kr for t in range(T)]
    assert oracle_lib.histogram(idx, Nr).tolist() == [4, 3, 7, 0]


def test_empty_batch(oracle_lib):
    idx = np.zeros((0, 8), np.int32)
    offsets, order = oracle_lib.expert_order(idx, 16)
    assert offsets.tolist() == [0] * 17 and order.size == 0
    assert oracle_lib.histogram(idx, 16).tolist() == [0] * 16


@pytest.mark.parametrize("T,Kr,Nr,seed", [(1, 1, 1, 0), (33, 4, 16, 1), (200, 8, 32, 2), (64, 8, 256, 3)])
def test_random_matches_brute_force(oracle_lib, T, Kr, Nr, seed):
    rng = np.random.default_rng(seed)
    # distinct experts per token, as a top-k selection gives; skewed toward
    # low indices so some experts repeat across many tokens and some are empty
    idx = np.stack([rng.choice(Nr, size=Kr, replace=False, p=np.arange(Nr, 0, -1) / (Nr * (Nr + 1) / 2))
                    for _ in range(T)]).astype(np.int32)
    offsets, order = oracle_lib.expert_order(idx, Nr)
    b_off, b_ord = brute_order(idx, Nr)
    assert offsets.tolist() == b_off.tolist()
    assert order.tolist() == b_ord.tolist()
    # the histogram is the run lengths, and every assignment appears once
    assert oracle_lib.histogram(idx, Nr).tolist() == np.diff(b_off).tolist()
    assert sorted(order.tolist()) == list(range(T * Kr))
    # the same order as sorting the triples (expert, token, slot)
    triples = sorted((int(idx[t, k]), t, k) for t in range(T) for k in range(Kr))
    assert order.tolist() == [t * Kr + k for _, t, k in triples]
