"""Pins of the oracle's greedy verification (CPU only).

Standard greedy speculative verification, which H-Spec follows (evolve.pub review of
H-Spec, Frequently asked questions): the target's argmax at each of the K+1 block
positions, the longest prefix of drafts equal to it, the target's token after that
prefix, and the context advanced by the accepted drafts plus that token.  The
expected values are built with numpy (argmax, cumulative product of the matches) on
inputs constructed so that each case is known.
"""
import numpy as np
import torch

import oracle


def expected(logits, drafts):
    lg = np.asarray(logits, dtype=np.float64)
    t = np.argmax(np.where(np.isnan(lg), -np.inf, lg), axis=-1)  # first max: lowest id on ties
    K = drafts.shape[1]
    match = (np.asarray(drafts) == t[:, :K]).astype(np.int64)
    acc = np.cumprod(match, axis=1).sum(axis=1)
    nxt = t[np.arange(len(acc)), acc]
    return acc, nxt


def test_accepted_length_is_the_matching_prefix():
    g = torch.Generator().manual_seed(0)
    C, K, V = 9, 6, 77
    lg = torch.randn(C, K + 1, V, generator=g)
    t = lg.argmax(-1)
    drafts = torch.randint(0, V, (C, K), generator=g)
    for c in range(C):  # request c accepts exactly min(c, K) drafts
        L = min(c, K)
        drafts[c, :L] = t[c, :L]
        if L < K:
            drafts[c, L] = (t[c, L] + 1) % V
    acc, nxt, ctx = oracle.verify_greedy(lg, drafts, torch.full((C,), 100))
    assert acc.tolist() == [min(c, K) for c in range(C)]
    assert nxt.tolist() == [int(t[c, min(c, K)]) for c in range(C)]
    assert ctx.tolist() == [100 + min(c, K) + 1 for c in range(C)]
    e_acc, e_nxt = expected(lg, drafts)
    assert np.array_equal(acc, e_acc) and np.array_equal(nxt, e_nxt)


def test_all_accepted_takes_the_bonus_token_and_random_drafts_agree_with_numpy():
    g = torch.Generator().manual_seed(1)
    C, K, V = 5, 4, 300
    lg = torch.randn(C, K + 1, V, generator=g).to(torch.bfloat16)
    t = lg.float().argmax(-1)
    drafts = t[:, :K].clone()
    acc, nxt, _ = oracle.verify_greedy(lg, drafts)
    assert acc.tolist() == [K] * C and nxt.tolist() == t[:, K].tolist()
    rnd = torch.randint(0, 3, (C, K), generator=g)  # mostly rejected at position 0
    acc2, nxt2, _ = oracle.verify_greedy(lg, rnd)
    e_acc, e_nxt = expected(lg.float(), rnd)
    assert np.array_equal(acc2, e_acc) and np.array_equal(nxt2, e_nxt)


def test_ties_take_the_lowest_id_and_nan_never_wins():
    K, V = 2, 10
    lg = torch.zeros(1, K + 1, V)
    lg[0, 0, 7] = lg[0, 0, 3] = 5.0          # tie: id 3
    lg[0, 1, 2] = float("nan")
    lg[0, 1, 8] = 1.0                        # NaN skipped: id 8
    lg[0, 2] = float("nan")                  # no number in the row: -1
    acc, nxt, _ = oracle.verify_greedy(lg, torch.tensor([[3, 8]]))
    assert acc.tolist() == [2] and nxt.tolist() == [-1]
    acc, nxt, _ = oracle.verify_greedy(lg, torch.tensor([[7, 8]]))
    assert acc.tolist() == [0] and nxt.tolist() == [3]


def test_single_draft():
    lg = torch.tensor([[[0.0, 2.0, 1.0], [3.0, 0.0, 0.0]]])
    acc, nxt, _ = oracle.verify_greedy(lg, torch.tensor([[1]]))
    assert acc.tolist() == [1] and nxt.tolist() == [0]
    acc, nxt, _ = oracle.verify_greedy(lg, torch.tensor([[2]]))
    assert acc.tolist() == [0] and nxt.tolist() == [1]
