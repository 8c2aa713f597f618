"""The fold pins must catch plausible mistakes in the oracle's folding
functions.  Each mutant wraps the real function with one planted error (on
the CPU, in test code only); the battery of checks from the fold pins (hand
trees, brute force, the prefill recurrence, decoding on from the folded
state) must reject every mutant and accept the real functions."""
import numpy as np
import pytest

from oracle import gdn
from tests.test_oracle_pins import random_problem


def plist(*steps):
    return [np.asarray(s, dtype=np.int64) for s in steps]


def cad_mutant(mutation):
    def fn(parents, t, max_depth):
        D, shared = gdn.common_ancestor_depth(parents, t, max_depth)
        if mutation == "one_too_deep":
            D = np.minimum(D + 1, min(t, max_depth))
        elif mutation == "ignores_cap":
            D, shared = gdn.common_ancestor_depth(parents, t, t)
        elif mutation == "own_depth_never":
            W_t = np.asarray(parents[t - 1]).shape[-1]
            if W_t == 1:
                D = np.minimum(D, t - 1)
        elif mutation == "any_two_beams":
            par = [np.asarray(p) for p in parents]
            anc = gdn.ancestry_walk(par, t)
            D = np.array([t - 1 if anc.shape[1] > 1 and (anc[r, 0] == anc[r, 1]).all() else D[r]
                          for r in range(anc.shape[0])])
        shared = [np.asarray(s)[:d] if len(s) >= d else np.concatenate([s, np.zeros(d - len(s), np.int64)])
                  for s, d in zip(shared, D)]
        return D, shared
    return fn


def fold_mutant(mutation):
    def fn(S0, steps, D):
        D = np.asarray(D, dtype=np.int64)
        if mutation == "one_depth_short":
            return gdn.fold_state(S0, steps, np.maximum(D - 1, 0))
        if mutation == "prompt_state":
            return gdn.to_f64(S0).copy()
        if mutation == "wrong_beam":
            res = gdn.beam_decode_fullstate(S0, steps[:int(D.max())], keep_states=True)
            out = gdn.to_f64(S0).copy()
            _, shared = gdn.common_ancestor_depth([s["parents"] for s in steps], len(steps), len(steps))
            for r in range(out.shape[0]):
                d = int(D[r])
                if d > 0:
                    Wd = res[d - 1]["S"].shape[1]
                    out[r] = res[d - 1]["S"][r, (shared[r][d - 1] + 1) % Wd]
            return out
        return gdn.fold_state(S0, steps, D)
    return fn


def battery(cad, fold):
    fails = []
    # hand-built trees
    cases = [
        (plist([[0, 0, 0]], [[1, 1, 1]], [[0, 2, 1]]), 3, 3, 1),
        (plist([[0, 0, 0]], [[1, 1, 1]], [[2, 2, 2]]), 3, 3, 2),
        (plist([[0, 0, 0]], [[1, 1, 1]], [[2, 2, 2]]), 3, 1, 1),
        (plist([[0, 0, 0]], [[0, 1, 2]]), 2, 2, 0),
        (plist([[0, 0, 0]], [[2]]), 2, 2, 2),
        (plist([[0, 0], [0, 0]], [[1, 1], [0, 1]], [[0, 1], [1, 1]]), 3, 3, None),
    ]
    for parents, t, md, want in cases:
        D, _ = cad(parents, t, md)
        if want is None:
            if D.tolist() != [1, 2]:
                fails.append("hand")
        elif D.tolist() != [want]:
            fails.append("hand")
    # brute force on random trees
    rng = np.random.default_rng(3)
    for _ in range(4):
        Ws = [int(rng.integers(1, 5)) for _ in range(5)]
        pl, Wp = [], 1
        for W in Ws:
            pl.append(rng.integers(0, Wp, size=(2, W)))
            Wp = W
        t = len(Ws)
        D, _ = cad(pl, t, t)
        for r in range(2):
            paths = []
            for b in range(Ws[-1]):
                node, path = b, [b]
                for s in range(t - 1, 0, -1):
                    node = int(pl[s][r, node])
                    path.append(node)
                paths.append(path[::-1])
            d = 0
            while d < t and all(pa[d] == paths[0][d] for pa in paths):
                d += 1
            if D[r] != d:
                fails.append("brute")
    # single beam: the prefill recurrence
    S0, steps = random_problem(3, R=1, H=2, dk=6, dv=5, Ws=(1, 1, 1))
    for d in (1, 2, 3):
        got = fold(S0, steps, [d])
        k = np.concatenate([s["k"] for s in steps[:d]], axis=1)
        v = np.concatenate([s["v"] for s in steps[:d]], axis=1)
        a = np.concatenate([s["alpha"] for s in steps[:d]], axis=1)
        b = np.concatenate([s["beta"] for s in steps[:d]], axis=1)
        if np.abs(got - gdn.prefill(k, v, a, b, S_init=S0)).max() > 1e-12:
            fails.append("prefill")
            break
    # decoding on from the folded state equals the unfolded decode
    S0, steps = random_problem(12, R=1, H=2, dk=5, dv=4, Ws=(4, 5, 3, 6, 4), parents="uniform")
    steps[2]["parents"] = np.full_like(steps[2]["parents"], 1)
    full = gdn.beam_decode_fullstate(S0, steps)
    Sf = fold(S0, steps[:4], [2])
    cont = gdn.beam_decode_fullstate(S0, steps[2:], S_prev=np.repeat(Sf[:, None], steps[1]["parents"].shape[1], 1))
    if np.abs(cont[-1]["o"] - full[-1]["o"]).max() > 1e-12:
        fails.append("continue")
    return sorted(set(fails))


def test_real_functions_pass_the_battery():
    assert battery(gdn.common_ancestor_depth, gdn.fold_state) == []


@pytest.mark.parametrize("mutation", ["one_too_deep", "ignores_cap", "own_depth_never", "any_two_beams"])
def test_battery_rejects_shared_depth_mutant(mutation):
    assert battery(cad_mutant(mutation), gdn.fold_state) != []


@pytest.mark.parametrize("mutation", ["one_depth_short", "prompt_state", "wrong_beam"])
def test_battery_rejects_fold_state_mutant(mutation):
    assert battery(gdn.common_ancestor_depth, fold_mutant(mutation)) != []
