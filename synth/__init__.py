"""Seeded synthetic inputs for the shared-state GDN beam decode.

This module only draws random numbers and casts them to the storage types the
decode operator consumes.  It holds none of the method's arithmetic: no state
update, no projection, no replay.  Both the fp64 oracle (``oracle/``) and the
CUDA path read the very same tensors produced here, so the two sides consume
identical bits.

Workload shapes follow the OneLA pages (OneLA abstract; evolve.pub review,
"Summary" and key claims on section 4.2 / 4.3): one shared prompt-derived
state per request, beam width W in the hundreds, prompts of 1K / 5K tokens and
3-7 decode steps.  The pages' model and data are proprietary, so every tensor
here is synthetic with the distributions listed below.

Draw order (fixed, per request r, generator seeded with
``SeedSequence([workload.seed_id, r, 0])``):
  1. the prompt: L tokens of (k, v, alpha, beta) per head, or, when
     ``L_prompt == 0``, S0 entries drawn directly from N(0, 0.1^2);
  2. for each decode step t = 1..T: q, k, v, alpha, beta, parents.

Distributions: q, k ~ N(0, I) then L2-normalised in fp64; v ~ N(0, 1);
alpha ~ U(0.85, 0.999) (passed to the operator as g = fp32(ln alpha));
beta = sigmoid(N(0, 1)); parents uniform over the previous step's beams or
truncated Zipf(s) over the previous step's beam rank (P(p=r) ~ (r+1)^-s).
At step 1 the previous "beam set" is the prompt root alone, so every parent
is 0.
"""
from __future__ import annotations

import dataclasses
from typing import Dict, List, Optional

import numpy as np
import torch

__all__ = [
    "Workload",
    "WORKLOADS",
    "workload",
    "zipf_probs",
    "draw_prompt",
    "draw_s0_direct",
    "draw_decode",
    "cast_state",
    "cast_vec",
]


@dataclasses.dataclass(frozen=True)
class Workload:
    """One synthetic workload: shapes, dtypes and the parent distribution."""

    name: str
    R: int            # concurrent requests, each with its own S0
    H: int            # heads
    d_k: int
    d_v: int
    W: int            # beams per request after step 1
    T: int            # decode steps
    L_prompt: int     # prompt tokens used to build S0 (0: S0 drawn directly)
    s0_dtype: str     # "f32" | "bf16"
    qkv_dtype: str    # "f32" | "bf16"
    parents: str      # "uniform" | "zipf" | "mixed" (even r uniform, odd r zipf)
    zipf_s: float = 1.1
    seed_id: int = 0

    def replace(self, **kw) -> "Workload":
        return dataclasses.replace(self, **kw)

    @property
    def units(self) -> int:
        """Beam-head decode steps in one whole T-step decode."""
        return self.R * self.W * self.H * self.T


# The workloads.  ``seed_id`` keeps every workload on its own random stream.
WORKLOADS: Dict[str, Workload] = {
    # Tiny correctness case: all fp32, S0 drawn directly, uniform parents.
    "tiny": Workload("tiny", R=1, H=2, d_k=64, d_v=64, W=8, T=3, L_prompt=0,
                     s0_dtype="f32", qkv_dtype="f32", parents="uniform",
                     seed_id=0),
    # Per-step operator with a 1K-token prompt state.
    "op1k": Workload("op1k", R=1, H=16, d_k=128, d_v=128, W=256, T=3,
                     L_prompt=1024, s0_dtype="f32", qkv_dtype="bf16",
                     parents="zipf", seed_id=1),
    # Long prompt, deeper decode (the headline workload) and its bf16-S0 twin.
    "long5k": Workload("long5k", R=1, H=16, d_k=128, d_v=128, W=256, T=7,
                       L_prompt=5120, s0_dtype="f32", qkv_dtype="bf16",
                       parents="zipf", seed_id=2),
    "long5k_bf16": Workload("long5k_bf16", R=1, H=16, d_k=128, d_v=128, W=256,
                            T=7, L_prompt=5120, s0_dtype="bf16",
                            qkv_dtype="bf16", parents="zipf", seed_id=2),
}
# Beam-width sweep, T=5, 1K prompt.
for _w in (64, 128, 256, 512, 1024):
    WORKLOADS[f"wsweep{_w}"] = Workload(
        f"wsweep{_w}", R=1, H=16, d_k=128, d_v=128, W=_w, T=5, L_prompt=1024,
        s0_dtype="f32", qkv_dtype="bf16", parents="zipf", seed_id=3)


def shape_sweep_workload(R: int, H: int, d: int, W: int, T: int) -> Workload:
    """Multi-request operator-shape sweep member (1K prompt per request)."""
    return Workload(f"sweep_R{R}_H{H}_d{d}_W{W}_T{T}", R=R, H=H, d_k=d, d_v=d,
                    W=W, T=T, L_prompt=1024, s0_dtype="f32", qkv_dtype="bf16",
                    parents="mixed" if R > 1 else "zipf", seed_id=4)


# The d = 256 point of the operator-shape sweep by name (profiling runs).
WORKLOADS["sweep_R1_H16_d256_W256_T7"] = shape_sweep_workload(1, 16, 256, 256, 7)


def workload(name: str) -> Workload:
    return WORKLOADS[name]


def zipf_probs(n: int, s: float) -> np.ndarray:
    """Truncated Zipf over ranks 0..n-1: P(r) proportional to (r+1)^-s."""
    w = np.arange(1, n + 1, dtype=np.float64) ** (-s)
    return w / w.sum()


def _rng(wl: Workload, r: int) -> np.random.Generator:
    return np.random.default_rng(np.random.SeedSequence([wl.seed_id, r, 0]))


def _unit_rows(x: np.ndarray) -> np.ndarray:
    return x / np.linalg.norm(x, axis=-1, keepdims=True)


def _sigmoid(x: np.ndarray) -> np.ndarray:
    return 1.0 / (1.0 + np.exp(-x))


def _draw_prompt_one(rng, wl: Workload):
    L, H = wl.L_prompt, wl.H
    k = _unit_rows(rng.standard_normal((L, H, wl.d_k)))
    v = rng.standard_normal((L, H, wl.d_v))
    alpha = rng.uniform(0.85, 0.999, size=(L, H))
    beta = _sigmoid(rng.standard_normal((L, H)))
    return k, v, alpha, beta


def _parent_kind(wl: Workload, r: int) -> str:
    if wl.parents == "mixed":
        return "uniform" if r % 2 == 0 else "zipf"
    return wl.parents


def _draw_step_one(rng, wl: Workload, r: int, W_prev: int, W: int):
    H = wl.H
    q = _unit_rows(rng.standard_normal((W, H, wl.d_k)))
    k = _unit_rows(rng.standard_normal((W, H, wl.d_k)))
    v = rng.standard_normal((W, H, wl.d_v))
    alpha = rng.uniform(0.85, 0.999, size=(W, H))
    beta = _sigmoid(rng.standard_normal((W, H)))
    kind = _parent_kind(wl, r)
    if W_prev == 1:
        parents = np.zeros(W, dtype=np.int64)
    elif kind == "uniform":
        parents = rng.integers(0, W_prev, size=W)
    elif kind == "zipf":
        parents = rng.choice(W_prev, size=W, p=zipf_probs(W_prev, wl.zipf_s))
    else:
        raise ValueError(f"unknown parent distribution {kind!r}")
    return q, k, v, alpha, beta, parents


def draw_prompt(wl: Workload):
    """Prompt tokens for every request, fp64: k [R][L][H][d_k] (unit rows),
    v [R][L][H][d_v], alpha [R][L][H], beta [R][L][H].

    The decode inputs of each request are drawn after its prompt from the same
    stream, so this function consumes nothing that ``draw_decode`` needs; it
    re-seeds per request.
    """
    if wl.L_prompt <= 0:
        raise ValueError("workload draws S0 directly; use draw_s0_direct")
    ks, vs, als, bes = [], [], [], []
    for r in range(wl.R):
        k, v, a, b = _draw_prompt_one(_rng(wl, r), wl)
        ks.append(k); vs.append(v); als.append(a); bes.append(b)
    return np.stack(ks), np.stack(vs), np.stack(als), np.stack(bes)


def draw_s0_direct(wl: Workload) -> np.ndarray:
    """S0 entries drawn from N(0, 0.1^2), fp64, [R][H][d_v][d_k]."""
    out = []
    for r in range(wl.R):
        rng = _rng(wl, r)
        out.append(0.1 * rng.standard_normal((wl.H, wl.d_v, wl.d_k)))
    return np.stack(out)


def cast_vec(x: np.ndarray, dtype: str) -> torch.Tensor:
    """fp64 -> fp32 (round to nearest even) -> bf16 (round to nearest even)."""
    t = torch.from_numpy(np.ascontiguousarray(x, dtype=np.float32))
    if dtype == "f32":
        return t
    if dtype == "bf16":
        return t.to(torch.bfloat16)
    raise ValueError(dtype)


def cast_state(S: np.ndarray, dtype: str) -> torch.Tensor:
    """Cast an fp64 state to the stored S0 type (same rounding as cast_vec)."""
    return cast_vec(S, dtype)


def draw_decode(wl: Workload, W_schedule: Optional[List[int]] = None):
    """Decode inputs for steps t = 1..T as a list of dicts of CPU tensors:

    q, k  [R][W][H][d_k]   qkv dtype (unit rows before the cast)
    v     [R][W][H][d_v]   qkv dtype
    g     [R][W][H]        fp32, g = fp32(ln alpha)
    beta  [R][W][H]        fp32
    parents [R][W]         int32, each in [0, W_prev)
    W_prev, W              ints

    ``W_schedule`` optionally gives the beam count of every step (default: W at
    every step); the previous count of step 1 is always 1 (the prompt root).
    """
    sched = list(W_schedule) if W_schedule is not None else [wl.W] * wl.T
    if len(sched) != wl.T:
        raise ValueError("W_schedule must have T entries")
    rngs = []
    for r in range(wl.R):
        rng = _rng(wl, r)
        # Skip past the prompt draws so that the decode stream follows them.
        if wl.L_prompt > 0:
            _draw_prompt_one(rng, wl)
        else:
            rng.standard_normal((wl.H, wl.d_v, wl.d_k))
        rngs.append(rng)
    steps = []
    W_prev = 1
    for t in range(wl.T):
        W = sched[t]
        per = [_draw_step_one(rngs[r], wl, r, W_prev, W) for r in range(wl.R)]
        q = np.stack([p[0] for p in per])
        k = np.stack([p[1] for p in per])
        v = np.stack([p[2] for p in per])
        alpha = np.stack([p[3] for p in per])
        beta = np.stack([p[4] for p in per])
        parents = np.stack([p[5] for p in per])
        steps.append({
            "q": cast_vec(q, wl.qkv_dtype),
            "k": cast_vec(k, wl.qkv_dtype),
            "v": cast_vec(v, wl.qkv_dtype),
            "g": torch.from_numpy(np.log(alpha).astype(np.float32)),
            "beta": torch.from_numpy(beta.astype(np.float32)),
            "parents": torch.from_numpy(parents.astype(np.int32)),
            "W_prev": W_prev,
            "W": W,
        })
        W_prev = W
    return steps


def distinct_ancestors(parent_list: List[np.ndarray], t: int) -> int:
    """Number of distinct (depth, beam) records reachable from the beams of
    step t (1-based) through the parent arrays of one request: the records at
    depths 1..t-1 that some step-t beam replays.  Pure index bookkeeping used
    by the byte model; it walks parents, no arithmetic of the method."""
    if t <= 1:
        return 0
    total = 0
    frontier = np.unique(np.asarray(parent_list[t - 1]))  # depth t-1 beams
    for depth in range(t - 1, 0, -1):
        total += frontier.size
        if depth > 1:
            frontier = np.unique(np.asarray(parent_list[depth - 1])[frontier])
    return total

