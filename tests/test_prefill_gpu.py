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

Tensor-core handles (bf16 k and v, d_k = d_v in {64, 128}) take the prompt in
chunks of 64 tokens.  There every tensor-core operand that is not a bf16
value enters as three bf16 terms (relative residual about 2^-24, as fp32
rounding) with fp32 accumulation, and the segments are combined in fp32, so
the same tolerance holds; the tests below check that this path ran (its
launch count) and hold it to the oracle at that tolerance.
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
        assert h.last_launches() == 4  # the chunked tensor-core path
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


def _tc_prefill(wl, dev, segments):
    import linear_attention_beam_shared_b200 as L
    h = L.BeamDecoder(wl.R, wl.H, wl.d_k, wl.d_v, wl.W, wl.T, wl.s0_dtype, wl.qkv_dtype, kernel=L.ONELA_KERNEL_TC)
    try:
        h.prefill_segments(segments)
        h.prefill(dev["k"], dev["v"], dev["g"], dev["beta"])
        launches = h.last_launches()
        S = h.prompt_state()
        torch.cuda.synchronize()
        assert h.status() == 0
        return S.cpu(), launches
    finally:
        h.close()


@pytest.mark.parametrize("s0", ["f32", "bf16"])
@pytest.mark.parametrize("shape,segments", [
    ((1, 2, 128, 1), 0), ((1, 2, 128, 63), 0), ((1, 2, 128, 64), 1), ((2, 3, 128, 65), 2),
    ((1, 1, 64, 200), 3), ((2, 2, 64, 130), 0), ((1, 2, 128, 1000), 16), ((1, 3, 128, 777), 5),
])
def test_prefill_tc_chunked(shape, segments, s0):
    """The chunked tensor-core prefill (four launches: the per-chunk solve,
    the segment chains, their combination, the S0 image): a single token, a
    ragged last chunk, one exact chunk, one token past it, several requests
    and heads, d = 64 (rows past d_v zero in the 128-row MMA), more segments
    asked for than the prompt has chunks, an uneven split into segments."""
    R, H, d, Lp = shape
    wl = synth.Workload("pftc", R=R, H=H, d_k=d, d_v=d, W=8, T=3, L_prompt=Lp, s0_dtype=s0, qkv_dtype="bf16",
                        parents="uniform", seed_id=13)
    dev, ref = prompt_inputs(wl)
    S, launches = _tc_prefill(wl, dev, segments)
    assert launches == 4
    check_state(S, gdn.prefill(ref["k"], ref["v"], ref["a"], ref["b"]), s0)


def test_prefill_tc_segments_agree():
    """Every way of cutting the prompt into segments gives the state within
    the fp32 tolerance of the others (the combination through the transition
    matrices is exact up to rounding)."""
    wl = synth.Workload("pftc2", R=1, H=2, d_k=128, d_v=128, W=8, T=3, L_prompt=1500, s0_dtype="f32",
                        qkv_dtype="bf16", parents="uniform", seed_id=14)
    dev, ref = prompt_inputs(wl)
    S_ref = gdn.prefill(ref["k"], ref["v"], ref["a"], ref["b"])
    base, _ = _tc_prefill(wl, dev, 1)
    scale = max(1.0, float(np.abs(S_ref).max()))
    for segs in (2, 4, 7, 12):
        S, _ = _tc_prefill(wl, dev, segs)
        check_state(S, S_ref, "f32")
        assert float((S - base).abs().max()) <= 2 * REL_TOL * scale


def test_prefill_tc_matches_token_path():
    """The chunked path and the token-by-token path of a SIMT handle build
    the same state up to rounding."""
    import linear_attention_beam_shared_b200 as L
    wl = synth.Workload("pftc3", R=2, H=2, d_k=64, d_v=64, W=8, T=3, L_prompt=300, s0_dtype="f32",
                        qkv_dtype="bf16", parents="uniform", seed_id=15)
    dev, ref = prompt_inputs(wl)
    S_tc, _ = _tc_prefill(wl, dev, 0)
    S_tok, h = gpu_prefill(wl, dev, kernel=L.ONELA_KERNEL_SIMT)
    try:
        assert h.last_launches() == 1
    finally:
        h.close()
    scale = max(1.0, float(S_tok.abs().max()))
    assert float((S_tc - S_tok).abs().max()) <= 2 * REL_TOL * scale


def test_prefill_tc_bad_segments():
    import linear_attention_beam_shared_b200 as L
    h = L.BeamDecoder(1, 1, 64, 64, 8, 3, "f32", "bf16")
    try:
        for bad in (-1, 17):
            with pytest.raises(L.OnelaError):
                h.prefill_segments(bad)
    finally:
        h.close()
