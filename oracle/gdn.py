"""Plain fp64 CPU oracle for one shared-state GDN beam-decode step.

TEST INFRASTRUCTURE.  Only the test suite, the package smoke check and the
CPU-baseline leg of the benchmark may import this module; the product path
never does.  It shares no code with the CUDA library.

What it computes (OneLA, evolve.pub review, key claims on section 3.2,
equations 2-4, and the abstract): every beam b of a request holds a Gated
DeltaNet state that starts from the request's shared prompt-derived state S0
and is advanced once per decode step,

    S_t = alpha_t S_{t-1} + delta_t k_t^T,
    delta_t = beta_t (v_t - alpha_t S_{t-1} k_t),
    o_t = S_t q_t,

where S_{t-1} is the state of the beam's parent (the beam it was expanded
from).  The pages state that the method is exact, with no approximation
(review, key claims on section 3.2), so this oracle is that plain definition
written out: the FullState baseline's semantics (review, Summary and report
preview "Scope & Claims"), a full d_v x d_k state per
beam, copied from the parent at every step, and the output taken literally as
S_t q_t.  Nothing is blocked, fused or reordered beyond numpy's own matrix
products.

Functions
---------
prefill               GDN recurrence from the zero state over prompt tokens.
gdn_sequential        one beam, T steps (W = 1 everywhere), outputs per step.
beam_decode_fullstate the beam tree with a full state per beam (the oracle).
beam_decode_replay    the projection-replay formulation (records + ancestry),
                      in fp64; used only to check "replay == full state".
ancestry_walk         pointer walk over the parent arrays (depth-ordered
                      ancestor beam indices of every beam).
common_ancestor_depth the deepest depth whose ancestor every beam of a step
                      shares (the folding extension).
fold_state            the full state of that shared ancestor, taken from the
                      full-state beam tree (the folding extension's result).

Conventions: alpha = exp(g) in fp64 from the fp32 g the operator receives;
every input is first converted exactly to fp64 (``to_f64``).
"""
from __future__ import annotations

from typing import Dict, List, Sequence

import numpy as np

__all__ = [
    "to_f64",
    "alpha_of",
    "prefill",
    "gdn_sequential",
    "beam_decode_fullstate",
    "beam_decode_replay",
    "ancestry_walk",
    "common_ancestor_depth",
    "fold_state",
]


def to_f64(x) -> np.ndarray:
    """Exact conversion of a stored tensor (fp32 / bf16 / numpy) to fp64."""
    try:
        import torch
        if isinstance(x, torch.Tensor):
            return x.detach().to(torch.float64).cpu().numpy()
    except ImportError:  # pragma: no cover
        pass
    return np.asarray(x, dtype=np.float64)


def alpha_of(g) -> np.ndarray:
    """The decay gate alpha = exp(g), in fp64 from the stored g."""
    return np.exp(to_f64(g))


def prefill(k, v, alpha, beta, S_init=None) -> np.ndarray:
    """Run the GDN recurrence from S_init (default: zero) over L tokens.

    k [..., L, H, d_k], v [..., L, H, d_v], alpha/beta [..., L, H] (fp64).
    Returns S [..., H, d_v, d_k].  Leading dims (e.g. requests) are batched.
    """
    k = to_f64(k); v = to_f64(v); alpha = to_f64(alpha); beta = to_f64(beta)
    lead = k.shape[:-3]
    L, H, dk = k.shape[-3:]
    dv = v.shape[-1]
    S = np.zeros(lead + (H, dv, dk)) if S_init is None else to_f64(S_init).copy()
    for l in range(L):
        kl = k[..., l, :, :]
        vl = v[..., l, :, :]
        al = alpha[..., l, :][..., None]
        bl = beta[..., l, :][..., None]
        u = np.einsum("...ij,...j->...i", S, kl)          # S_{l-1} k_l
        delta = bl * (vl - al * u)
        S = al[..., None] * S + delta[..., :, None] * kl[..., None, :]
    return S


def gdn_sequential(S0, q, k, v, alpha, beta):
    """One beam for T steps.  S0 [H][d_v][d_k]; q/k [T][H][d_k]; v [T][H][d_v];
    alpha/beta [T][H].  Returns (o [T][H][d_v], delta [T][H][d_v], S_T)."""
    S = to_f64(S0).copy()
    q = to_f64(q); k = to_f64(k); v = to_f64(v)
    alpha = to_f64(alpha); beta = to_f64(beta)
    outs, deltas = [], []
    for t in range(q.shape[0]):
        a = alpha[t][:, None]
        u = np.einsum("hij,hj->hi", S, k[t])
        delta = beta[t][:, None] * (v[t] - a * u)
        S = a[..., None] * S + delta[:, :, None] * k[t][:, None, :]
        outs.append(np.einsum("hij,hj->hi", S, q[t]))
        deltas.append(delta)
    return np.stack(outs), np.stack(deltas), S


def _step_inputs(step: Dict) -> tuple:
    return (to_f64(step["q"]), to_f64(step["k"]), to_f64(step["v"]),
            alpha_of(step["g"]) if "g" in step else to_f64(step["alpha"]),
            to_f64(step["beta"]), np.asarray(step["parents"], dtype=np.int64))


def beam_decode_fullstate(S0, steps: Sequence[Dict], S_prev=None,
                          keep_states: bool = False) -> List[Dict[str, np.ndarray]]:
    """The oracle: a full fp64 state per beam, copied from the parent.

    S0: [R][H][d_v][d_k] (any stored type; converted exactly to fp64).
    steps[t]: q, k [R][W][H][d_k]; v [R][W][H][d_v]; g (or alpha), beta
    [R][W][H]; parents [R][W] with values in [0, W_prev), W_prev = 1 at t = 1.
    S_prev: optional [R][W_prev][H][d_v][d_k], the states of the beams the
    first given step expands (default: S0 as the single root).
    Returns per step: o, delta [R][W][H][d_v] and alpha [R][W][H] (fp64), and
    with keep_states the states S_t [R][W][H][d_v][d_k] as "S".
    """
    S0 = to_f64(S0)
    R = S0.shape[0]
    S_prev = S0[:, None] if S_prev is None else to_f64(S_prev)   # [R][W_prev][H][d_v][d_k]
    out = []
    for step in steps:
        q, k, v, alpha, beta, parents = _step_inputs(step)
        if parents.min(initial=0) < 0 or parents.max(initial=0) >= S_prev.shape[1]:
            raise ValueError("parent index out of range")
        # FullState: copy the parent's state into the child.
        S = S_prev[np.arange(R)[:, None], parents]            # [R][W][H][dv][dk]
        a = alpha[..., None]                                   # [R][W][H][1]
        u = np.einsum("rwhij,rwhj->rwhi", S, k)                # S_{t-1} k_t
        delta = beta[..., None] * (v - a * u)
        S = a[..., None] * S + delta[..., :, None] * k[..., None, :]
        o = np.einsum("rwhij,rwhj->rwhi", S, q)                # S_t q_t
        out.append({"o": o, "delta": delta, "alpha": alpha})
        if keep_states:
            out[-1]["S"] = S
        S_prev = S
    return out


def ancestry_walk(parent_list: Sequence, t: int) -> np.ndarray:
    """Ancestors of every beam of step t (1-based), found by walking parent
    pointers one depth at a time.

    parent_list[s-1] holds the parents of step s ([R][W_s] or [W_s]).
    Returns anc [..., W_t, t-1] int64 with anc[..., b, j] = index of the beam
    at depth j+1 on the path from the root to beam b of step t.
    """
    par = [np.asarray(p, dtype=np.int64) for p in parent_list]
    cur = par[t - 1]                       # parents of step-t beams: depth t-1
    shape = cur.shape
    anc = np.zeros(shape + (max(t - 1, 0),), dtype=np.int64)
    if t <= 1:
        return anc
    node = cur.copy()
    for depth in range(t - 1, 0, -1):
        anc[..., depth - 1] = node
        if depth > 1:
            prev = par[depth - 1]          # parents of step-`depth` beams
            if prev.ndim == 1:
                node = prev[node]
            else:
                node = np.take_along_axis(prev, node, axis=-1)
    return anc


def common_ancestor_depth(parent_list: Sequence, t: int, max_depth: int):
    """Per request, the deepest depth D <= max_depth at which every beam of
    step t has the same ancestor, and that ancestor at each depth 1..D.

    The beam of depth t itself counts as its own ancestor at depth t, so a
    step that kept one beam shares depth t.  parent_list[s-1] holds the
    parents [R][W_s] of step s.  Returns (D [R] int64, list of R int64 arrays
    of length D_r with the shared ancestor at depths 1..D_r).
    """
    par = [np.asarray(p, dtype=np.int64) for p in parent_list]
    R, W_t = par[t - 1].shape
    # Path of every beam of step t, depth 1 .. t (its own index last).
    paths = np.concatenate([ancestry_walk(par, t), np.broadcast_to(np.arange(W_t), (R, W_t))[..., None]],
                           axis=-1)
    D = np.zeros(R, dtype=np.int64)
    shared = []
    for r in range(R):
        d = 0
        while d < min(t, max_depth) and len(set(paths[r, :, d].tolist())) == 1:
            d += 1
        D[r] = d
        shared.append(paths[r, 0, :d].copy())
    return D, shared


def fold_state(S0, steps: Sequence[Dict], D) -> np.ndarray:
    """The state each request's decode replays from once depths 1..D[r] are
    folded: the full state of the shared ancestor at depth D[r] (S0 where
    D[r] = 0), read off the full-state beam tree.  [R][H][d_v][d_k] fp64."""
    S0 = to_f64(S0)
    D = np.asarray(D, dtype=np.int64)
    out = S0.copy()
    if D.max(initial=0) == 0:
        return out
    res = beam_decode_fullstate(S0, steps[:int(D.max())], keep_states=True)
    t = len(steps)
    _, shared = common_ancestor_depth([s["parents"] for s in steps], t, t)
    for r in range(S0.shape[0]):
        d = int(D[r])
        if d > 0:
            if len(shared[r]) < d:
                raise ValueError("no shared ancestor at that depth")
            out[r] = res[d - 1]["S"][r, shared[r][d - 1]]
    return out


def beam_decode_replay(S0, steps: Sequence[Dict]) -> List[Dict[str, np.ndarray]]:
    """Projection replay in fp64: never forms a per-beam state.

    Each beam keeps only its transition record (alpha_t, delta_t, k_t).  For a
    beam of step t whose ancestors carry records j = 1..t-1,
        S_{t-1} x = G (S0 x) + sum_j w_j (k_j . x) delta_j,
        w_j = prod_{i>j} alpha_i,  G = prod_{i=1}^{t-1} alpha_i,
    for x in {k_t, q_t}; then delta_t = beta_t (v_t - alpha_t S_{t-1} k_t) and
    o_t = alpha_t S_{t-1} q_t + delta_t (k_t . q_t).
    Used only to check that replay equals the full-state oracle.
    """
    S0 = to_f64(S0)
    records = []          # per depth: alpha [R][W][H], delta [R][W][H][dv], k [R][W][H][dk]
    parent_list = []
    out = []
    for t, step in enumerate(steps, start=1):
        q, k, v, alpha, beta, parents = _step_inputs(step)
        parent_list.append(parents)
        anc = ancestry_walk(parent_list, t)                  # [R][W][t-1]
        R, W, H = alpha.shape
        rr = np.arange(R)[:, None]
        uk = np.einsum("rhij,rwhj->rwhi", S0, k)
        uq = np.einsum("rhij,rwhj->rwhi", S0, q)
        G = np.ones((R, W, H))
        acc_k = np.zeros_like(uk)
        acc_q = np.zeros_like(uq)
        for j in range(t - 1, 0, -1):                        # depth j record
            a_rec, d_rec, k_rec = records[j - 1]
            bj = anc[..., j - 1]                             # [R][W]
            a_j = a_rec[rr, bj]                              # [R][W][H]
            d_j = d_rec[rr, bj]                              # [R][W][H][dv]
            k_j = k_rec[rr, bj]                              # [R][W][H][dk]
            w = G                                            # prod over depths > j
            acc_k += (w * np.einsum("rwhj,rwhj->rwh", k_j, k))[..., None] * d_j
            acc_q += (w * np.einsum("rwhj,rwhj->rwh", k_j, q))[..., None] * d_j
            G = G * a_j
        uk = G[..., None] * uk + acc_k
        uq = G[..., None] * uq + acc_q
        a = alpha[..., None]
        delta = beta[..., None] * (v - a * uk)
        o = a * uq + delta * np.einsum("rwhj,rwhj->rwh", k, q)[..., None]
        records.append((alpha, delta, k))
        out.append({"o": o, "delta": delta, "alpha": alpha})
    return out
