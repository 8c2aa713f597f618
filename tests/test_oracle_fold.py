"""Pins for the oracle's folding functions (an extension of the method: the
evolve.pub review's Summary and Weaknesses name the replay cost that grows
with decode depth).  Checked against hand-built beam trees, a brute-force
path walk, the GDN recurrence run as a prefill, and the exactness of
continuing a decode from the folded state.
"""
import numpy as np
import pytest

from oracle import gdn
from tests.test_oracle_pins import random_problem


def plist(*steps):
    return [np.asarray(s, dtype=np.int64) for s in steps]


# ------------------------------------------------------- hand-built trees
@pytest.mark.parametrize("parents,t,max_depth,D,shared", [
    # depth-1 ancestor 1 shared; depth-2 ancestors 0, 2, 1 differ
    (plist([[0, 0, 0]], [[1, 1, 1]], [[0, 2, 1]]), 3, 3, 1, [1]),
    # every step-3 beam descends from beam 2 of depth 2, itself from beam 1
    (plist([[0, 0, 0]], [[1, 1, 1]], [[2, 2, 2]]), 3, 3, 2, [1, 2]),
    (plist([[0, 0, 0]], [[1, 1, 1]], [[2, 2, 2]]), 3, 1, 1, [1]),
    (plist([[0, 0, 0]], [[1, 1, 1]], [[2, 2, 2]]), 3, 0, 0, []),
    # the beams split at the root
    (plist([[0, 0, 0]], [[0, 1, 2]]), 2, 2, 0, []),
    # one beam kept: its own depth is shared too
    (plist([[0, 0, 0]], [[2]]), 2, 2, 2, [2, 0]),
    (plist([[0]], [[0]], [[0]]), 3, 3, 3, [0, 0, 0]),
])
def test_common_ancestor_depth_hand_trees(parents, t, max_depth, D, shared):
    got_D, got_shared = gdn.common_ancestor_depth(parents, t, max_depth)
    assert got_D.tolist() == [D]
    assert got_shared[0].tolist() == shared


def test_common_ancestor_depth_per_request():
    parents = plist([[0, 0], [0, 0]], [[1, 1], [0, 1]], [[0, 1], [1, 1]])
    D, shared = gdn.common_ancestor_depth(parents, 3, 3)
    # request 0: paths [1,0,0], [1,1,1] share depth 1 only; request 1:
    # paths [1,1,0], [1,1,1] share depths 1 and 2
    assert D.tolist() == [1, 2]
    assert shared[0].tolist() == [1] and shared[1].tolist() == [1, 1]
    D, _ = gdn.common_ancestor_depth(plist([[0, 0], [0, 0]], [[1, 1], [0, 1]]), 2, 2)
    assert D.tolist() == [1, 0]


@pytest.mark.parametrize("seed", range(6))
def test_common_ancestor_depth_brute_force(seed):
    """Random trees (some with a forced bottleneck) against a path walk on a
    child -> parent dictionary."""
    rng = np.random.default_rng(seed)
    Ws = [int(rng.integers(1, 6)) for _ in range(6)]
    R = 3
    pl, Wp = [], 1
    for s, W in enumerate(Ws):
        p = rng.integers(0, Wp, size=(R, W))
        if s == 3:
            p[1] = int(rng.integers(0, Wp))   # request 1 narrows to one parent
        pl.append(p)
        Wp = W
    t = len(Ws)
    D, shared = gdn.common_ancestor_depth(pl, t, t)
    for r in range(R):
        up = {(s + 1, b): (s, int(pl[s][r, b])) for s in range(t) for b in range(Ws[s])}
        paths = []
        for b in range(Ws[-1]):
            node, path = (t, b), []
            while node[0] >= 1:
                path.append(node[1])
                node = up[node]
            paths.append(path[::-1])
        d = 0
        while d < t and all(pa[d] == paths[0][d] for pa in paths):
            d += 1
        assert D[r] == d
        assert shared[r].tolist() == paths[0][:d]


# ------------------------------------------------------- the folded state
def test_fold_state_of_a_single_beam_is_the_prefill_recurrence():
    """W = 1 throughout: the folded state at depth D is the GDN recurrence
    from S0 over the first D tokens, run by the oracle's prefill."""
    S0, steps = random_problem(3, R=2, H=2, dk=6, dv=5, Ws=(1, 1, 1, 1))
    for D in range(5):
        got = gdn.fold_state(S0, steps, [D, max(D - 1, 0)])
        for r, d in enumerate([D, max(D - 1, 0)]):
            if d == 0:
                np.testing.assert_array_equal(got[r], S0[r])
                continue
            k = np.concatenate([s["k"][r:r + 1] for s in steps[:d]], axis=1)
            v = np.concatenate([s["v"][r:r + 1] for s in steps[:d]], axis=1)
            a = np.concatenate([s["alpha"][r:r + 1] for s in steps[:d]], axis=1)
            b = np.concatenate([s["beta"][r:r + 1] for s in steps[:d]], axis=1)
            ref = gdn.prefill(k, v, a, b, S_init=S0[r:r + 1])
            np.testing.assert_allclose(got[r], ref[0], rtol=0, atol=1e-13)


def bottleneck(steps, at, beam=0):
    """Make every beam of step `at` (0-based) a child of one beam, so that the
    beams of every later step share their ancestors at depths 1..at."""
    steps[at]["parents"] = np.full_like(steps[at]["parents"], beam)
    return steps


@pytest.mark.parametrize("seed", range(4))
def test_decoding_on_from_the_folded_state_is_exact(seed):
    """Fold after step t_f at the shared depth, then continue: every output of
    the later steps equals the unfolded decode's (fp64, rounding only).  The
    folded state is handed to every beam of the folded depth; only the
    descendants of the shared ancestor reach the steps compared."""
    S0, steps = random_problem(10 + seed, R=2, H=2, dk=7, dv=5, Ws=(4, 5, 3, 6, 4, 5), parents="uniform")
    steps = bottleneck(steps, 2, beam=seed % 5)      # step 3: all children of one beam
    t_f = 4
    D, shared = gdn.common_ancestor_depth([s["parents"] for s in steps[:t_f]], t_f, t_f)
    assert (D >= 2).all()
    full = gdn.beam_decode_fullstate(S0, steps)
    for Dm in range(1, int(D.min()) + 1):
        Sf = gdn.fold_state(S0, steps[:t_f], [Dm, Dm])
        W_D = steps[Dm - 1]["parents"].shape[1]
        S_prev = np.repeat(Sf[:, None], W_D, axis=1)
        cont = gdn.beam_decode_fullstate(S0, steps[Dm:], S_prev=S_prev)
        for t in range(t_f, len(steps)):             # steps t_f + 1 .. T (0-based t_f ..)
            np.testing.assert_allclose(cont[t - Dm]["o"], full[t]["o"], rtol=0, atol=1e-12)
            np.testing.assert_allclose(cont[t - Dm]["delta"], full[t]["delta"], rtol=0, atol=1e-12)


def test_folding_a_wrong_ancestor_is_detected():
    """The identity above is sensitive: the state of a beam that is not the
    shared ancestor gives different outputs."""
    S0, steps = random_problem(21, R=1, H=1, dk=5, dv=4, Ws=(4, 4, 4, 4), parents="uniform")
    steps = bottleneck(steps, 1, beam=2)
    full = gdn.beam_decode_fullstate(S0, steps, keep_states=True)
    wrong = full[0]["S"][:, 1]                       # depth-1 beam 1, not the shared beam 2
    cont = gdn.beam_decode_fullstate(S0, steps[1:], S_prev=np.repeat(wrong[:, None], 4, axis=1))
    assert np.abs(cont[-1]["o"] - full[-1]["o"]).max() > 1e-3
    right = gdn.fold_state(S0, steps[:2], [1])
    np.testing.assert_array_equal(right, full[0]["S"][:, 2])


def test_s_prev_default_is_the_prompt_root():
    S0, steps = random_problem(5, Ws=(3, 4))
    a = gdn.beam_decode_fullstate(S0, steps)
    b = gdn.beam_decode_fullstate(S0, steps, S_prev=S0[:, None])
    for x, y in zip(a, b):
        np.testing.assert_array_equal(x["o"], y["o"])


def test_fold_state_rejects_a_depth_without_a_shared_ancestor():
    S0, steps = random_problem(6, Ws=(3, 3, 3))
    steps[1]["parents"] = np.array([[0, 1, 2]])
    steps[2]["parents"] = np.array([[0, 1, 2]])       # paths [0,0,0], [1,1,1], [2,2,2]
    with pytest.raises(ValueError):
        gdn.fold_state(S0, steps, [1])
