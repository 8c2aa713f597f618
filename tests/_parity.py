"""Helpers shared by the GPU parity tests: build inputs from the seeded
generator, run the CUDA path through the C ABI, run the oracle on the same
tensors, and compare."""
from __future__ import annotations

import functools
from typing import Dict, List, Optional

import numpy as np
import torch

import synth
from oracle import cref, gdn

# Max-abs tolerances on o and delta against the fp64 oracle (bf16 S0 / fp32 S0).
TOL = {"bf16": 1e-3, "f32": 2e-5}
# alpha = expf(g) on the GPU vs exp(g) in fp64: a few fp32 ulps at alpha < 1.
TOL_ALPHA = 4e-7


@functools.lru_cache(maxsize=None)
def _prompt_state_f64(wl: synth.Workload) -> np.ndarray:
    if wl.L_prompt > 0:
        k, v, a, b = synth.draw_prompt(wl)
        return gdn.prefill(k, v, a, b)
    return synth.draw_s0_direct(wl)


def prompt_state_f64(wl: synth.Workload) -> np.ndarray:
    """S0 in fp64 for a workload: the oracle's prefill over its prompt, or
    drawn directly.  Depends only on the seed and the shapes, so the fp32 and
    bf16 twins of a workload share it."""
    return _prompt_state_f64(wl.replace(name="prompt", s0_dtype="f32", qkv_dtype="f32", T=1, W=1,
                                        parents="uniform"))


def prompt_state(wl: synth.Workload) -> torch.Tensor:
    return synth.cast_state(prompt_state_f64(wl), wl.s0_dtype)


def to_dev(steps, device="cuda"):
    return [{k: (v.to(device) if isinstance(v, torch.Tensor) else v) for k, v in s.items()} for s in steps]


def run_gpu(S0: torch.Tensor, steps: List[Dict], qkv_dtype: str, kernel: int,
            T_max: Optional[int] = None, W_max: Optional[int] = None, read_back=True,
            s0_split: int = 0, flags: int = 0, chunks: Optional[List[int]] = None):
    """Decode on the GPU through the C ABI.  chunks = None: one
    onela_decode_step call per step; else onela_decode_steps calls over
    consecutive runs of chunks[0], chunks[1], ... steps (a chunk of 1 is a
    onela_decode_step call)."""
    import linear_attention_beam_shared_b200 as L
    R, H, dv, dk = S0.shape
    s0_dtype = "bf16" if S0.dtype == torch.bfloat16 else "f32"
    T = len(steps)
    W_max = W_max or max(s["W"] for s in steps)
    dec = L.BeamDecoder(R, H, dk, dv, W_max, T_max or T, s0_dtype, qkv_dtype, kernel=kernel,
                        s0_split=s0_split, flags=flags)
    try:
        dsteps = to_dev(steps)          # every input resident before the first step
        dec.set_prompt_state(S0.cuda())
        outs = []
        if chunks is None:
            for s in dsteps:
                o = dec.step(s["q"], s["k"], s["v"], s["g"], s["beta"], s["parents"])
                outs.append(o)
        else:
            assert sum(chunks) == T
            i = 0
            for c in chunks:
                if c == 1:
                    s = dsteps[i]
                    outs.append(dec.step(s["q"], s["k"], s["v"], s["g"], s["beta"], s["parents"]))
                else:
                    outs += dec.steps(dsteps[i:i + c])
                i += c
        assert dec.status() == 0
        res = []
        for t, o in enumerate(outs, start=1):
            r = {"o": o.cpu()}
            if read_back:
                a, d, kr = dec.records(t)
                r["alpha"] = a.cpu().permute(0, 2, 1).contiguous()          # [R][W][H]
                r["delta"] = d.cpu().permute(0, 2, 1, 3).contiguous()       # [R][W][H][dv]
                r["k"] = kr.cpu().permute(0, 2, 1, 3).contiguous()          # [R][W][H][dk]
                r["anc"] = dec.ancestry(t).cpu()
            res.append(r)
        return res, dec.kernel
    finally:
        dec.close()


def oracle(S0: torch.Tensor, steps: List[Dict], use_c=True):
    if use_c:
        return cref.beam_decode_fullstate(S0, steps)
    return gdn.beam_decode_fullstate(S0, steps)


def compare(gpu, ref, steps, s0_dtype: str, check_records=True):
    """Max-abs errors; asserts the tolerances and bit-exact indexing."""
    tol = TOL[s0_dtype]
    worst = {"o": 0.0, "delta": 0.0, "alpha": 0.0}
    plist = [s["parents"].numpy() for s in steps]
    for t, (g, r, s) in enumerate(zip(gpu, ref, steps), start=1):
        eo = float(np.abs(g["o"].double().numpy() - r["o"]).max())
        worst["o"] = max(worst["o"], eo)
        assert np.isfinite(g["o"].numpy()).all()
        if check_records and "delta" in g:
            ed = float(np.abs(g["delta"].double().numpy() - r["delta"]).max())
            worst["delta"] = max(worst["delta"], ed)
            ea = float(np.abs(g["alpha"].double().numpy() - gdn.alpha_of(s["g"])).max())
            worst["alpha"] = max(worst["alpha"], ea)
            assert torch.equal(g["k"], s["k"]), f"k record differs at step {t}"
            anc_ref = gdn.ancestry_walk(plist, t)
            assert np.array_equal(g["anc"].numpy().astype(np.int64), anc_ref), f"ancestry differs at step {t}"
    assert worst["o"] <= tol, f"o max-abs error {worst['o']:.3e} > {tol:.1e}"
    assert worst["delta"] <= tol, f"delta max-abs error {worst['delta']:.3e} > {tol:.1e}"
    assert worst["alpha"] <= TOL_ALPHA, f"alpha error {worst['alpha']:.3e}"
    return worst


def custom_steps(seed, R, H, dk, dv, Ws, qkv_dtype="bf16", parents="zipf", fixed=None):
    """Seeded steps with an explicit beam schedule (shapes outside the named
    workloads).  Draws through the same generator module."""
    wl = synth.Workload("custom", R=R, H=H, d_k=dk, d_v=dv, W=max(Ws), T=len(Ws), L_prompt=0,
                        s0_dtype="f32", qkv_dtype=qkv_dtype, parents=parents, seed_id=1000 + seed)
    steps = synth.draw_decode(wl, W_schedule=list(Ws))
    if fixed is not None:
        for t, s in enumerate(steps):
            if t > 0:
                s["parents"] = torch.from_numpy(fixed(t, s["W_prev"], s["W"], R).astype(np.int32))
    S0 = synth.draw_s0_direct(wl)
    return wl, S0, steps
