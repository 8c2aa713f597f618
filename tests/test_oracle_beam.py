"""Pins of the beam-selection oracle (oracle/beam.py) against things other
than itself: a brute-force ordering of Python tuples built one candidate at a
time, a hand-worked example, and the cases the ordering rule fixes (fp32
rounding ties, signed zeros, NaN, -inf, W = all candidates)."""
import math

import numpy as np
import pytest

from oracle import beam


def brute_force(beam_score, logp, W):
    R, W_prev, C = logp.shape
    out = []
    for r in range(R):
        cands = []
        for b in range(W_prev):
            for c in range(C):
                s = float(np.float32(beam_score[r, b]) + np.float32(logp[r, b, c]))  # one fp32 rounding
                if s == 0.0:
                    s = 0.0
                cands.append((1 if math.isnan(s) else 0, 0.0 if math.isnan(s) else -s, b * C + c, s))
        cands.sort(key=lambda x: x[:3])
        out.append([(f // C, f % C, s) for _, _, f, s in cands[:W]])
    return out


@pytest.mark.parametrize("R,W_prev,C,W,levels", [(1, 4, 5, 7, 3), (3, 6, 4, 24, 5), (2, 9, 3, 5, 100),
                                                  (1, 1, 17, 17, 4)])
def test_matches_brute_force_with_many_ties(R, W_prev, C, W, levels):
    rng = np.random.default_rng(R * 100 + W)
    bs = rng.integers(0, levels, (R, W_prev)).astype(np.float32) * 0.5
    lp = -rng.integers(0, levels, (R, W_prev, C)).astype(np.float32) * 0.25
    parent, token, score = beam.select_beams(bs, lp, W)
    ref = brute_force(bs, lp, W)
    for r in range(R):
        assert [(int(p), int(t)) for p, t in zip(parent[r], token[r])] == [(b, c) for b, c, _ in ref[r]]
        np.testing.assert_array_equal(score[r], np.array([s for _, _, s in ref[r]], np.float32))


def test_hand_worked_example():
    # child scores: beam 0 -> [0.5, -0.2, 0.5], beam 1 -> [1.0, -1.0, -inf]
    bs = np.array([[0.0, -1.0]], np.float32)
    lp = np.array([[[0.5, -0.2, 0.5], [2.0, 0.0, -np.inf]]], np.float32)
    parent, token, score = beam.select_beams(bs, lp, 4)
    assert parent.tolist() == [[1, 0, 0, 0]]
    assert token.tolist() == [[0, 0, 2, 1]]
    assert score.tolist() == [[1.0, 0.5, 0.5, np.float32(-0.2)]]


def test_scores_are_rounded_to_fp32_before_ranking():
    # 1e8 + 1 and 1e8 + 2 are both 1e8 in fp32 (spacing 8): a tie, so the
    # smaller flat index (beam 0, child 0) comes first although 2 > 1.
    bs = np.array([[1e8]], np.float32)
    lp = np.array([[[1.0, 2.0]]], np.float32)
    parent, token, score = beam.select_beams(bs, lp, 2)
    assert token.tolist() == [[0, 1]]
    assert score.tolist() == [[1e8, 1e8]]


def test_signed_zeros_tie_and_nan_ranks_last():
    bs = np.zeros((1, 1), np.float32)
    lp = np.array([[[np.nan, -0.0, -np.inf, 0.0, -1.0]]], np.float32)
    parent, token, score = beam.select_beams(bs, lp, 5)
    assert token.tolist() == [[1, 3, 4, 2, 0]]  # -0 and +0 tie -> index order; -inf; then NaN
    assert np.isnan(score[0, 4]) and score[0, 3] == -np.inf


def test_all_candidates_is_a_full_sort():
    rng = np.random.default_rng(3)
    bs = rng.standard_normal((2, 5)).astype(np.float32)
    lp = rng.standard_normal((2, 5, 6)).astype(np.float32)
    parent, token, score = beam.select_beams(bs, lp, 30)
    for r in range(2):
        assert sorted(zip(parent[r], token[r])) == [(b, c) for b in range(5) for c in range(6)]
        assert np.all(np.diff(score[r]) <= 0)
