"""GPU parity of the prefill (onela_prefill, through the C ABI): the state
built on the device from a prompt against the fp64 oracle's prefill on the
same seeded, already-rounded inputs (k and v in the handle's qkv type, g and
beta in fp32, alpha = exp(g) taken in fp64 on the oracle side).

Tolerance: the kernel runs the recurrence in fp32.  Each token rounds every
state element a few times (a fused multiply-add and the dot product u), so
the error added per token is a few units of 2^-24 of the state's scale; the
gates (alpha <= 0.999) forget it over at most about 1000 tokens, and the
rounding errors of different tokens are independent, so the accumulated
error stays near sqrt(1000) x 2^-24 x max|S|, about 2e-6 x max|S|.  The test
allows 1e-5 x max(1, max|S|) (five times that) as max-abs error; a bf16 S0
is the fp32 result rounded once, so it may differ from the rounded oracle by
one bf16 unit where the fp32 value lies next to a rounding boundary.
"""
import numpy as np
import pytest
import torch

import synth
from oracle import gdn
from tests import _parity as P

pytestmark = pytest.mark.gpu

REL_TOL = 1e-5


def prompt_inputs(wl, L=None):
    """Prompt tokens of a workload in the handle's types (device tensors) and
    the fp64 arrays the oracle gets (the same rounded values)."""
    k, v, a, b = synth.draw_prompt(wl)
    if L is not None:
        k, v, a, b = k[:, :L], v[:, :L], a[:, :L], b[:, :L]
    kd = synth.cast_vec(k, wl.qkv_dtype)
    vd = synth.cast_vec(v, wl.qkv_dtype)
    g = torch.from_numpy(np.log(a)).float()
    beta = torch.from_numpy(b).float()
    ref = dict(k=kd.double().numpy(), v=vd.double().numpy(), a=np.exp(g.double().numpy()), b=beta.double().numpy())
    dev = dict(k=kd.cuda().contiguous(), v=vd.cuda().contiguous(), g=g.cuda().contiguous(), beta=beta.cuda().contiguous())
    return dev, ref


def gpu_prefill(wl, dev, kernel=0):
    import linear_attention_beam_shared_b200 as L
    h = L.BeamDecoder(wl.R, wl.H, wl.d_k, wl.d_v, wl.W, wl.T, wl.s0_dtype, wl.qkv_dtype, kernel=kernel)
    try:
        h.prefill(dev["k"], dev["v"], dev["g"], dev["beta"])
        S = h.prompt_state()
        torch.cuda.synchronize()
        assert h.status() == 0
        return S.cpu(), h
    except Exception:
        h.close()
        raise


def check_state(S_gpu, S_ref, s0_dtype):
    scale = max(1.0, float(np.abs(S_ref).max()))
    if s0_dtype == "f32":
        err = float(np.abs(S_gpu.double().numpy() - S_ref).max())
        print(f"prefill max-abs error {err:.3g} (state scale {scale:.3g})")
        assert err <= REL_TOL * scale, (err, scale)
    else:
        ref16 = synth.cast_state(S_ref, "bf16")
        diff = (S_gpu.float() - ref16.float()).abs()
        # one bf16 unit of the larger of the two, plus the fp32 error before
        # the rounding (which dominates for elements near zero)
        ulp = torch.maximum(S_gpu.float().abs(), ref16.float().abs()) * 2.0 ** -7
        assert bool((diff <= ulp + REL_TOL * scale).all()), float((diff - ulp).max())
        assert float((diff > 0).float().mean()) < 0.01  # almost every element identical


@pytest.mark.parametrize("qkv,s0", [("f32", "f32"), ("bf16", "f32"), ("bf16", "bf16"), ("f32", "bf16")])
@pytest.mark.parametrize("shape", [(2, 3, 64, 48, 77), (1, 2, 128, 128, 100), (1, 2, 256, 256, 40),
                                   (2, 1, 33, 33, 5), (1, 1, 7, 20, 1)])
def test_prefill_small(shape, qkv, s0):
    """Several tiles, a ragged last row block and token chunk, odd widths
    (plain copies of unaligned rows), a single token."""
    R, H, dk, dv, Lp = shape
    wl = synth.Workload("pf", R=R, H=H, d_k=dk, d_v=dv, W=8, T=3, L_prompt=Lp, s0_dtype=s0, qkv_dtype=qkv,
                        parents="uniform", seed_id=11)
    dev, ref = prompt_inputs(wl)
    S, h = gpu_prefill(wl, dev)
    h.close()
    check_state(S, gdn.prefill(ref["k"], ref["v"], ref["a"], ref["b"]), s0)


def test_prefill_single_token_closed_form():
    """From the zero state one token gives S = beta v k^T exactly (no gate)."""
    wl = synth.Workload("pf1", R=1, H=2, d_k=64, d_v=64, W=8, T=3, L_prompt=1, s0_dtype="f32", qkv_dtype="f32",
                        parents="uniform", seed_id=12)
    dev, ref = prompt_inputs(wl)
    S, h = gpu_prefill(wl, dev)
    h.close()
    closed = ref["b"][0, 0][:, None, None] * ref["v"][0, 0][:, :, None] * ref["k"][0, 0][:, None, :]
    np.testing.assert_allclose(S[0].double().numpy(), closed, rtol=1e-6, atol=1e-7)


@pytest.mark.parametrize("name", ["op1k", "long5k"])
def test_prefill_full_size_then_decode(name):
    """The workload's whole prompt (1024 or 5120 tokens, 16 heads, d = 128),
    then its decode from the device-built state against the oracle's decode
    from the same state."""
    wl = synth.workload(name)
    dev, ref = prompt_inputs(wl)
    S, h = gpu_prefill(wl, dev)
    try:
        check_state(S, gdn.prefill(ref["k"], ref["v"], ref["a"], ref["b"]), wl.s0_dtype)
        steps = synth.draw_decode(wl)
        ds = P.to_dev(steps)
        outs = [h.step(s["q"], s["k"], s["v"], s["g"], s["beta"], s["parents"]) for s in ds]
        torch.cuda.synchronize()
        assert h.status() == 0
        ref_out = P.oracle(S, steps)
        for t, (o, r) in enumerate(zip(outs, ref_out)):
            err = float(np.abs(o.double().cpu().numpy() - r["o"]).max())
            assert err <= P.TOL[wl.s0_dtype], (t + 1, err)
    finally:
        h.close()


def test_prefill_rewinds_the_decode():
    import linear_attention_beam_shared_b200 as L
    wl = synth.workload("tiny").replace(L_prompt=10)
    dev, _ = prompt_inputs(wl)
    S, h = gpu_prefill(wl, dev)
    try:
        steps = P.to_dev(synth.draw_decode(wl))
        h.step(steps[0]["q"], steps[0]["k"], steps[0]["v"], steps[0]["g"], steps[0]["beta"], steps[0]["parents"])
        assert L.onela_steps_done(h.h) == 1
        h.prefill(dev["k"], dev["v"], dev["g"], dev["beta"])
        assert L.onela_steps_done(h.h) == 0
        torch.testing.assert_close(h.prompt_state().cpu(), S, rtol=0, atol=0)
    finally:
        h.close()
