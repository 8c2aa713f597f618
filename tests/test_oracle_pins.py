"""Pins for the fp64 oracle: checks against facts that do not come from the
oracle itself (closed forms, exact rational arithmetic, the textbook matrix
form of the gated delta rule, invariants, brute force, a hand-worked example).

The method and its exactness claim: OneLA abstract and the evolve.pub review
(key claims on section 3.2, equations 2-4, which state that the replay
reproduces GDN exactly).
"""
import json
import os
from fractions import Fraction

import numpy as np
import pytest

import synth
from oracle import gdn

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def random_problem(seed, R=1, H=2, dk=8, dv=6, Ws=(5, 7, 4), parents="uniform",
                   alpha_range=(0.85, 0.999)):
    """Small fp64 problem with alpha given directly (no exp rounding)."""
    rng = np.random.default_rng(seed)
    S0 = 0.3 * rng.standard_normal((R, H, dv, dk))
    steps, Wp = [], 1
    for W in Ws:
        q = rng.standard_normal((R, W, H, dk))
        k = rng.standard_normal((R, W, H, dk))
        k /= np.linalg.norm(k, axis=-1, keepdims=True)
        q /= np.linalg.norm(q, axis=-1, keepdims=True)
        v = rng.standard_normal((R, W, H, dv))
        alpha = rng.uniform(*alpha_range, size=(R, W, H))
        beta = 1 / (1 + np.exp(-rng.standard_normal((R, W, H))))
        if Wp == 1:
            par = np.zeros((R, W), dtype=np.int64)
        elif parents == "uniform":
            par = rng.integers(0, Wp, size=(R, W))
        else:
            par = np.stack([rng.choice(Wp, size=W, p=synth.zipf_probs(Wp, 1.1)) for _ in range(R)])
        steps.append(dict(q=q, k=k, v=v, alpha=alpha, beta=beta, parents=par))
        Wp = W
    return S0, steps


# ---------------------------------------------------------------- closed form
def test_single_step_closed_form_exact_rational():
    """t = 1: o = alpha S0 q + beta (v - alpha S0 k)(k . q) and
    delta = beta (v - alpha S0 k), evaluated in exact rational arithmetic on
    dyadic inputs (d = 2, three beams from the root)."""
    F = Fraction
    S0 = [[F(1, 2), F(-3, 4)], [F(5, 8), F(1, 4)]]
    beams = [
        dict(k=[F(1), F(1, 2)], q=[F(-1, 2), F(3, 4)], v=[F(1), F(-2)], a=F(3, 4), b=F(1, 2)),
        dict(k=[F(-1, 4), F(1)], q=[F(1), F(1)], v=[F(0), F(1, 2)], a=F(7, 8), b=F(1, 4)),
        dict(k=[F(3, 2), F(-1, 2)], q=[F(1, 8), F(-1)], v=[F(-1), F(3)], a=F(1, 2), b=F(3, 4)),
    ]

    def mv(S, x):
        return [S[i][0] * x[0] + S[i][1] * x[1] for i in range(2)]

    exp_o, exp_d = [], []
    for bm in beams:
        Sk = mv(S0, bm["k"])
        Sq = mv(S0, bm["q"])
        kq = bm["k"][0] * bm["q"][0] + bm["k"][1] * bm["q"][1]
        d = [bm["b"] * (bm["v"][i] - bm["a"] * Sk[i]) for i in range(2)]
        exp_d.append(d)
        exp_o.append([bm["a"] * Sq[i] + d[i] * kq for i in range(2)])
    step = dict(
        q=np.array([[[[float(x) for x in bm["q"]]] for bm in beams]]),
        k=np.array([[[[float(x) for x in bm["k"]]] for bm in beams]]),
        v=np.array([[[[float(x) for x in bm["v"]]] for bm in beams]]),
        alpha=np.array([[[float(bm["a"])] for bm in beams]]),
        beta=np.array([[[float(bm["b"])] for bm in beams]]),
        parents=np.zeros((1, 3), dtype=np.int64))
    S0f = np.array([[[[float(x) for x in row] for row in S0]]])
    for fn in (gdn.beam_decode_fullstate, gdn.beam_decode_replay):
        out = fn(S0f, [step])[0]
        for b in range(3):
            for i in range(2):
                assert abs(out["o"][0, b, 0, i] - float(exp_o[b][i])) <= 1e-15
                assert abs(out["delta"][0, b, 0, i] - float(exp_d[b][i])) <= 1e-15


def test_golden_scalar_two_steps():
    """Hand-worked scalar example (tests/golden/scalar_two_steps.json)."""
    with open(os.path.join(GOLDEN, "scalar_two_steps.json")) as f:
        gold = json.load(f)
    S0 = np.array(gold["S0"]).reshape(1, 1, 1, 1)
    steps = []
    for st in gold["steps"]:
        W = len(st["parents"])
        steps.append(dict(
            q=np.array(st["q"]).reshape(1, W, 1, 1), k=np.array(st["k"]).reshape(1, W, 1, 1),
            v=np.array(st["v"]).reshape(1, W, 1, 1), alpha=np.array(st["alpha"]).reshape(1, W, 1),
            beta=np.array(st["beta"]).reshape(1, W, 1), parents=np.array([st["parents"]])))
    for fn in (gdn.beam_decode_fullstate, gdn.beam_decode_replay):
        out = fn(S0, steps)
        for st, o in zip(gold["steps"], out):
            assert o["o"].reshape(-1).tolist() == st["o"]
            assert o["delta"].reshape(-1).tolist() == st["delta"]


# ------------------------------------------------------ textbook gated delta
def textbook_chain(S0, steps):
    """Gated delta rule in its usual matrix form, one beam (W = 1):
    S_t = S_{t-1} (alpha_t (I - beta_t k_t k_t^T)) + beta_t v_t k_t^T, o_t = S_t q_t."""
    S = S0[0].copy()                       # [H][dv][dk]
    outs = []
    for st in steps:
        H, dk = st["k"].shape[2], st["k"].shape[3]
        o = np.zeros((H, S.shape[1]))
        for h in range(H):
            k = st["k"][0, 0, h]; q = st["q"][0, 0, h]; v = st["v"][0, 0, h]
            a = st["alpha"][0, 0, h]; b = st["beta"][0, 0, h]
            M = a * (np.eye(dk) - b * np.outer(k, k))
            S[h] = S[h] @ M + b * np.outer(v, k)
            o[h] = S[h] @ q
        outs.append(o)
    return outs


def test_textbook_gated_delta_rule_single_lineage():
    S0, steps = random_problem(3, R=1, H=3, dk=7, dv=5, Ws=(1, 1, 1, 1, 1, 1))
    ref = textbook_chain(S0, steps)
    for fn in (gdn.beam_decode_fullstate, gdn.beam_decode_replay):
        out = fn(S0, steps)
        for o_ref, o in zip(ref, out):
            np.testing.assert_allclose(o["o"][0, 0], o_ref, atol=1e-12, rtol=0)


def test_w1_equals_sequential_routine():
    S0, steps = random_problem(4, R=1, H=2, dk=9, dv=9, Ws=(1,) * 5)
    o_seq, d_seq, _ = gdn.gdn_sequential(
        S0[0], np.stack([s["q"][0, 0] for s in steps]), np.stack([s["k"][0, 0] for s in steps]),
        np.stack([s["v"][0, 0] for s in steps]), np.stack([s["alpha"][0, 0] for s in steps]),
        np.stack([s["beta"][0, 0] for s in steps]))
    out = gdn.beam_decode_fullstate(S0, steps)
    for t in range(5):
        np.testing.assert_allclose(out[t]["o"][0, 0], o_seq[t], atol=1e-12, rtol=0)
        np.testing.assert_allclose(out[t]["delta"][0, 0], d_seq[t], atol=1e-12, rtol=0)


def test_prefill_textbook_form():
    """prefill(...) from zero equals the textbook matrix-form recurrence."""
    rng = np.random.default_rng(5)
    L, H, dk, dv = 9, 2, 6, 4
    k = rng.standard_normal((L, H, dk)); k /= np.linalg.norm(k, axis=-1, keepdims=True)
    v = rng.standard_normal((L, H, dv))
    a = rng.uniform(0.85, 0.999, (L, H)); b = rng.uniform(0.1, 0.9, (L, H))
    S = gdn.prefill(k, v, a, b)
    ref = np.zeros((H, dv, dk))
    for l in range(L):
        for h in range(H):
            M = a[l, h] * (np.eye(dk) - b[l, h] * np.outer(k[l, h], k[l, h]))
            ref[h] = ref[h] @ M + b[l, h] * np.outer(v[l, h], k[l, h])
    np.testing.assert_allclose(S, ref, atol=1e-13, rtol=0)


def test_delta_rule_exact_recall():
    """alpha = 1, beta = 1 and a unit key: the delta rule stores v_t exactly
    at k_t, so with q_t = k_t the output is v_t (for any S0 and parent)."""
    S0, steps = random_problem(6, R=1, H=2, dk=8, dv=5, Ws=(4, 6))
    for st in steps:
        st["alpha"][:] = 1.0
        st["beta"][:] = 1.0
        st["q"] = st["k"].copy()
    for fn in (gdn.beam_decode_fullstate, gdn.beam_decode_replay):
        out = fn(S0, steps)
        for st, o in zip(steps, out):
            np.testing.assert_allclose(o["o"], st["v"], atol=1e-12, rtol=0)


# --------------------------------------------------------------- invariants
def test_identity_gate_no_write_keeps_s0():
    S0, steps = random_problem(7, R=2, H=2, dk=8, dv=6, Ws=(5, 7, 3))
    for st in steps:
        st["alpha"][:] = 1.0
        st["beta"][:] = 0.0
    out = gdn.beam_decode_fullstate(S0, steps)
    for st, o in zip(steps, out):
        assert np.all(o["delta"] == 0.0)
        ref = np.einsum("rhij,rwhj->rwhi", S0, st["q"])
        np.testing.assert_allclose(o["o"], ref, atol=1e-14, rtol=0)


def test_beta_zero_is_pure_gate_product():
    S0, steps = random_problem(8, R=1, H=3, dk=5, dv=4, Ws=(4, 6, 6, 5))
    for st in steps:
        st["beta"][:] = 0.0
    out = gdn.beam_decode_fullstate(S0, steps)
    plist = [st["parents"] for st in steps]
    for t, (st, o) in enumerate(zip(steps, out), start=1):
        W = st["alpha"].shape[1]
        for b in range(W):
            G = st["alpha"][0, b].copy()
            node = b
            for s in range(t, 1, -1):          # walk up: parent of step-s node
                node = plist[s - 1][0, node]
                G = G * steps[s - 2]["alpha"][0, node]
            ref = G[:, None] * np.einsum("hij,hj->hi", S0[0], st["q"][0, b])
            np.testing.assert_allclose(o["o"][0, b], ref, atol=1e-14, rtol=0)


def test_replay_equals_fullstate_small():
    for seed, kind in ((9, "uniform"), (10, "zipf"), (11, "zipf")):
        S0, steps = random_problem(seed, R=2, H=2, dk=12, dv=10, Ws=(6, 9, 9, 4, 11), parents=kind)
        a = gdn.beam_decode_fullstate(S0, steps)
        b = gdn.beam_decode_replay(S0, steps)
        for x, y in zip(a, b):
            np.testing.assert_allclose(x["o"], y["o"], atol=1e-12, rtol=0)
            np.testing.assert_allclose(x["delta"], y["delta"], atol=1e-12, rtol=0)


def test_replay_equals_fullstate_tiny_workload():
    wl = synth.workload("tiny")
    S0 = synth.cast_state(synth.draw_s0_direct(wl), wl.s0_dtype)
    steps = synth.draw_decode(wl)
    a = gdn.beam_decode_fullstate(S0, steps)
    b = gdn.beam_decode_replay(S0, steps)
    for x, y in zip(a, b):
        assert np.abs(x["o"] - y["o"]).max() <= 1e-12
        assert np.abs(x["delta"] - y["delta"]).max() <= 1e-12


def test_linearity_in_s0_and_v_is_exact():
    S0, steps = random_problem(12, R=1, H=2, dk=6, dv=6, Ws=(5, 5, 5))
    a = gdn.beam_decode_fullstate(S0, steps)
    steps2 = [dict(st, v=2.0 * st["v"]) for st in steps]
    b = gdn.beam_decode_fullstate(2.0 * S0, steps2)
    for x, y in zip(a, b):
        assert np.array_equal(2.0 * x["o"], y["o"])
        assert np.array_equal(2.0 * x["delta"], y["delta"])


def test_beam_relabeling_is_equivariant():
    """Permute the beams of step 2 and remap step 3's parents: outputs of
    step 2 permute, outputs of step 3 are unchanged."""
    S0, steps = random_problem(13, R=1, H=2, dk=6, dv=5, Ws=(4, 6, 5))
    perm = np.array([3, 0, 5, 1, 4, 2])          # new beam i = old beam perm[i]
    inv = np.argsort(perm)
    s2 = {key: (val[:, perm] if key != "parents" else val[:, perm]) for key, val in steps[1].items()}
    s3 = dict(steps[2], parents=inv[steps[2]["parents"]])
    a = gdn.beam_decode_fullstate(S0, steps)
    b = gdn.beam_decode_fullstate(S0, [steps[0], s2, s3])
    assert np.array_equal(a[1]["o"][:, perm], b[1]["o"])
    assert np.array_equal(a[2]["o"], b[2]["o"])


def test_oracle_rejects_bad_parent():
    S0, steps = random_problem(14, Ws=(3, 3))
    steps[1]["parents"][0, 1] = 3
    with pytest.raises(ValueError):
        gdn.beam_decode_fullstate(S0, steps)


# ----------------------------------------------------------------- ancestry
def brute_force_ancestry(parent_list, t):
    """Build the beam tree as explicit node objects, then read each path."""
    nodes = {(0, 0): None}                         # (depth, beam) -> parent node
    for s, par in enumerate(parent_list[:t], start=1):
        for b, p in enumerate(par):
            assert (s - 1, int(p)) in nodes
            nodes[(s, b)] = (s - 1, int(p))
    out = []
    for b in range(len(parent_list[t - 1])):
        path, node = [], nodes[(t, b)]
        while node != (0, 0):
            path.append(node[1])
            node = nodes[node]
        out.append(path[::-1])                     # depth 1 first
    return out


@pytest.mark.parametrize("kind", ["zeros", "identity", "reverse", "lineage", "uniform", "zipf"])
def test_ancestry_walk_matches_brute_force(kind):
    rng = np.random.default_rng(15)
    W, T = 9, 6
    plist = [np.zeros(W, dtype=np.int64)]
    for t in range(2, T + 1):
        if kind == "zeros":
            p = np.zeros(W, dtype=np.int64)
        elif kind == "identity":
            p = np.arange(W)
        elif kind == "reverse":
            p = np.arange(W)[::-1].copy()
        elif kind == "lineage":
            p = np.full(W, (t * 5) % W)
        elif kind == "uniform":
            p = rng.integers(0, W, W)
        else:
            p = rng.choice(W, size=W, p=synth.zipf_probs(W, 1.1))
        plist.append(p)
    for t in range(1, T + 1):
        anc = gdn.ancestry_walk(plist, t)
        ref = brute_force_ancestry(plist, t)
        assert anc.shape == (W, t - 1)
        assert anc.tolist() == ref


# ------------------------------------------------------------- C oracle twin
def test_c_oracle_matches_numpy_oracle():
    from oracle import cref
    for seed, Ws in ((16, (5, 7, 7, 3)), (17, (1, 9, 2, 8))):
        S0, steps = random_problem(seed, R=2, H=3, dk=10, dv=7, Ws=Ws)
        for st in steps:
            st["g"] = np.log(st.pop("alpha"))
        a = gdn.beam_decode_fullstate(S0, steps)
        b = cref.beam_decode_fullstate(S0, steps, nthreads=2)
        for x, y in zip(a, b):
            np.testing.assert_allclose(x["o"], y["o"], atol=1e-12, rtol=0)
            np.testing.assert_allclose(x["delta"], y["delta"], atol=1e-12, rtol=0)


def test_c_oracle_rejects_bad_parent():
    from oracle import cref
    S0, steps = random_problem(18, Ws=(3, 3))
    for st in steps:
        st["g"] = np.log(st.pop("alpha"))
    steps[1]["parents"][0, 0] = -1
    with pytest.raises(ValueError):
        cref.beam_decode_fullstate(S0, steps)
