"""The oracle's pins must catch plausible mistakes.  Each mutant below is a
copy of the full-state beam tree with one planted error (on the CPU, in test
code only); the battery of independent checks must reject every mutant and
accept the real oracle."""
import json
import os

import numpy as np
import pytest

from oracle import gdn
from tests.test_oracle_pins import GOLDEN, random_problem, textbook_chain


def make_fullstate(mutation=None):
    def fn(S0, steps):
        S0 = np.asarray(S0, dtype=np.float64)
        R = S0.shape[0]
        S_prev = S0[:, None]
        out = []
        for st in steps:
            q, k, v = st["q"], st["k"], st["v"]
            alpha, beta = st["alpha"], st["beta"]
            par = np.asarray(st["parents"])
            if mutation == "ignore_parent":
                par = np.minimum(np.arange(par.shape[1])[None, :], S_prev.shape[1] - 1).repeat(R, 0)
            S = S_prev[np.arange(R)[:, None], par]
            a = alpha[..., None]
            u = np.einsum("rwhij,rwhj->rwhi", S, k)
            if mutation == "no_alpha_in_delta":
                delta = beta[..., None] * (v - u)
            elif mutation == "delta_sign":
                delta = beta[..., None] * (a * u - v)
            else:
                delta = beta[..., None] * (v - a * u)
            if mutation == "no_alpha_decay":
                S_new = S + delta[..., :, None] * k[..., None, :]
            elif mutation == "transposed_outer":
                S_new = a[..., None] * S + k[..., :, None] * delta[..., None, :]
            elif mutation == "alpha_twice":
                S_new = a[..., None] * a[..., None] * S + delta[..., :, None] * k[..., None, :]
            else:
                S_new = a[..., None] * S + delta[..., :, None] * k[..., None, :]
            S_out = S if mutation == "output_old_state" else S_new
            o = np.einsum("rwhij,rwhj->rwhi", S_out, q)
            out.append({"o": o, "delta": delta})
            S_prev = S_new
        return out
    return fn


def battery(fn):
    failures = []
    # 1. hand-worked golden example
    with open(os.path.join(GOLDEN, "scalar_two_steps.json")) as f:
        gold = json.load(f)
    steps = []
    for st in gold["steps"]:
        W = len(st["parents"])
        steps.append(dict(
            q=np.array(st["q"]).reshape(1, W, 1, 1), k=np.array(st["k"]).reshape(1, W, 1, 1),
            v=np.array(st["v"]).reshape(1, W, 1, 1), alpha=np.array(st["alpha"]).reshape(1, W, 1),
            beta=np.array(st["beta"]).reshape(1, W, 1), parents=np.array([st["parents"]])))
    out = fn(np.array(gold["S0"]).reshape(1, 1, 1, 1), steps)
    if any(o["o"].reshape(-1).tolist() != st["o"] for st, o in zip(gold["steps"], out)):
        failures.append("golden")
    # 2. textbook matrix form on one lineage (square d so transposes run)
    S0, steps = random_problem(21, R=1, H=2, dk=6, dv=6, Ws=(1,) * 4)
    ref = textbook_chain(S0, steps)
    out = fn(S0, steps)
    if any(np.abs(o["o"][0, 0] - r).max() > 1e-12 for o, r in zip(out, ref)):
        failures.append("textbook")
    # 3. replay identity on a branching tree
    S0, steps = random_problem(22, R=1, H=2, dk=6, dv=6, Ws=(4, 6, 5), parents="zipf")
    ref = gdn.beam_decode_replay(S0, steps)
    out = fn(S0, steps)
    if any(np.abs(o["o"] - r["o"]).max() > 1e-12 for o, r in zip(out, ref)):
        failures.append("replay")
    return failures


MUTANTS = ["ignore_parent", "no_alpha_in_delta", "delta_sign", "no_alpha_decay",
           "transposed_outer", "alpha_twice", "output_old_state"]


def test_real_oracle_passes_battery():
    assert battery(gdn.beam_decode_fullstate) == []
    assert battery(make_fullstate(None)) == []


@pytest.mark.parametrize("mutation", MUTANTS)
def test_battery_rejects_mutant(mutation):
    assert battery(make_fullstate(mutation)) != []


@pytest.mark.parametrize("mutation", ["ignore_parent", "output_old_state", "delta_sign"])
def test_independent_pins_alone_reject_mutant(mutation):
    """Without the replay identity (oracle vs oracle), golden + textbook or a
    parent-sensitive gate-product check still catch each mutant."""
    fn = make_fullstate(mutation)
    fails = [f for f in battery(fn) if f != "replay"]
    if mutation == "ignore_parent":
        # parent mistakes need a branching tree: beta = 0 makes o a pure
        # product of the gates along the true ancestry
        S0, steps = random_problem(23, R=1, H=1, dk=4, dv=4, Ws=(4, 6, 5), parents="uniform")
        for st in steps:
            st["beta"][:] = 0.0
        out = fn(S0, steps)
        plist = [st["parents"] for st in steps]
        for t, (st, o) in enumerate(zip(steps, out), start=1):
            for b in range(st["alpha"].shape[1]):
                G, node = st["alpha"][0, b].copy(), b
                for s in range(t, 1, -1):
                    node = plist[s - 1][0, node]
                    G = G * steps[s - 2]["alpha"][0, node]
                ref = G[:, None] * np.einsum("hij,hj->hi", S0[0], st["q"][0, b])
                if np.abs(o["o"][0, b] - ref).max() > 1e-14:
                    fails.append("gate")
    assert fails
