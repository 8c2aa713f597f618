"""Plain CPU oracle for beam selection (the step after the decode step).

TEST INFRASTRUCTURE.  Only the test suite, the package smoke check and the
benchmark's CPU legs may import this module; the product path never does.  It
shares no code with the CUDA library.

What it computes: the pages describe large-beam decoding over a growing beam
tree (OneLA abstract: every step keeps a beam set and each beam's history is
a path of the tree) but do not spell out how the next beam set is chosen; the
plainest reading is the standard beam-search step.  For request r each
current beam b (of W_prev) has a cumulative score beam_score[r][b] and C
children c with log-probabilities logp[r][b][c]; the child's score is their
sum, formed in fp32 exactly as the device forms it (one rounding), and the W
children with the largest scores form the next beam set, best first.  Equal
scores go to the smaller flat index b * C + c; +0 and -0 are equal; NaN ranks
below every number.  The result: parent (= b), token (= c), score, each
[R][W].  Nothing more than numpy's sort is used.
"""
from __future__ import annotations

import numpy as np


def child_scores(beam_score, logp) -> np.ndarray:
    """fp32 [R][W_prev][C]: beam_score + logp with one fp32 rounding."""
    bs = np.asarray(beam_score, dtype=np.float32)
    lp = np.asarray(logp, dtype=np.float32)
    return (bs[:, :, None] + lp).astype(np.float32)


def select_beams(beam_score, logp, W: int):
    """Returns (parent int32 [R][W], token int32 [R][W], score fp32 [R][W])."""
    s = child_scores(beam_score, logp)
    R, W_prev, C = s.shape
    N = W_prev * C
    if not 1 <= W <= N:
        raise ValueError("need 1 <= W <= W_prev * C")
    flat_scores = s.reshape(R, N).astype(np.float64)
    parent = np.empty((R, W), np.int32)
    token = np.empty((R, W), np.int32)
    score = np.empty((R, W), np.float32)
    idx = np.arange(N)
    for r in range(R):
        x = flat_scores[r].copy()
        nan = np.isnan(x)
        x[nan] = 0.0
        x[x == 0.0] = 0.0   # -0 -> +0
        # Sort keys, last one primary: NaN last, then larger score first,
        # then the smaller flat index first.
        order = np.lexsort((idx, -x, nan))[:W]
        parent[r] = order // C
        token[r] = order % C
        score[r] = s.reshape(R, N)[r, order]
    return parent, token, score
