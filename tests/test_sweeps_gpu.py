"""GPU parity at the full sizes of the beam-width sweep and of the
multi-request shape grid.

The beam-width sweep (H=16, d=128, T=5, 1K prompt, W in {64 .. 1024}) is
compared element by element with the oracle.  The shape grid's large members
are run at full size on the GPU and checked on a sample of (request, head)
pairs, each recomputed alone by the oracle (every pair has its own S0 and
records, so a pair's outputs depend on nothing else); the ancestry rows are
compared in full."""
import numpy as np
import pytest
import torch

import synth
from oracle import cref, gdn
from tests import _parity as P

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("name", ["wsweep64", "wsweep128", "wsweep256", "wsweep512", "wsweep1024"])
def test_beam_width_sweep(name):
    import linear_attention_beam_shared_b200 as L
    wl = synth.workload(name)
    S0 = P.prompt_state(wl)
    steps = synth.draw_decode(wl)
    gpu, kind = P.run_gpu(S0, steps, wl.qkv_dtype, L.ONELA_KERNEL_AUTO, flags=L.ONELA_FLAG_PDL)
    assert kind == L.ONELA_KERNEL_TC
    P.compare(gpu, P.oracle(S0, steps), steps, wl.s0_dtype)


def _prompt_state_gpu(wl):
    """S0 by the GDN recurrence over the workload's prompt, in fp64 torch on
    the GPU (input synthesis only), cast to the workload's S0 type."""
    k, v, a, b = synth.draw_prompt(wl)
    dev = torch.device("cuda")
    k, v, a, b = (torch.from_numpy(x).to(dev) for x in (k, v, a, b))
    R, Lp, H, dk = k.shape
    S = torch.zeros((R, H, wl.d_v, dk), dtype=torch.float64, device=dev)
    for i in range(Lp):
        ki, vi, ai, bi = k[:, i], v[:, i], a[:, i, :, None], b[:, i, :, None]
        u = torch.einsum("rhij,rhj->rhi", S, ki)
        d = bi * (vi - ai * u)
        S = ai[..., None] * S + d[..., :, None] * ki[..., None, :]
    return synth.cast_state(S.cpu().numpy(), wl.s0_dtype)


def _slice(steps, r, h):
    out = []
    for s in steps:
        e = dict(s)
        for key in ("q", "k", "v"):
            e[key] = s[key][r:r + 1, :, h:h + 1].contiguous()
        for key in ("g", "beta"):
            e[key] = s[key][r:r + 1, :, h:h + 1].contiguous()
        e["parents"] = s["parents"][r:r + 1].contiguous()
        out.append(e)
    return out


@pytest.mark.parametrize("R,H,d,W,T,direct", [
    (32, 8, 64, 512, 7, False),
    (8, 32, 128, 512, 5, False),
    (1, 32, 256, 512, 7, False),
    (32, 32, 256, 512, 2, True),
    (1, 16, 128, 128, 1, False),
    (8, 16, 64, 256, 3, False),
    (4, 8, 256, 256, 5, True),
    (2, 16, 128, 128, 3, False),
])
def test_shape_grid_sampled(R, H, d, W, T, direct):
    """direct: S0 drawn directly (N(0, 0.1^2)) instead of the 1K-token
    prefill, which at R = H = 32, d = 256 would dominate the test's time."""
    import linear_attention_beam_shared_b200 as L
    wl = synth.shape_sweep_workload(R, H, d, W, T)
    S0 = synth.cast_state(synth.draw_s0_direct(wl.replace(L_prompt=0)), wl.s0_dtype) if direct \
        else _prompt_state_gpu(wl)
    steps = synth.draw_decode(wl)
    dec = L.BeamDecoder(R, H, d, d, W, T, wl.s0_dtype, wl.qkv_dtype, flags=L.ONELA_FLAG_PDL)
    rng = np.random.default_rng(R * 1000 + H * 10 + T)
    pairs = [(0, 0), (R - 1, H - 1)] + [(int(rng.integers(R)), int(rng.integers(H))) for _ in range(2)]
    try:
        dev_steps = P.to_dev(steps)
        dec.set_prompt_state(S0.cuda())
        outs = [dec.step(s["q"], s["k"], s["v"], s["g"], s["beta"], s["parents"]) for s in dev_steps]
        assert dec.status() == 0
        plist = [s["parents"].numpy() for s in steps]
        got = {pr: [] for pr in pairs}
        for t, o in enumerate(outs, start=1):
            assert np.array_equal(dec.ancestry(t).cpu().numpy().astype(np.int64), gdn.ancestry_walk(plist, t))
            _, dl, _ = dec.records(t)                 # delta [R][H][W][d]
            for (r, h) in pairs:
                got[(r, h)].append((o[r, :, h].cpu().double().numpy(), dl[r, h].cpu().double().numpy()))
            assert torch.isfinite(o).all()
        del outs
    finally:
        dec.close()
    tol = P.TOL[wl.s0_dtype]
    for (r, h) in pairs:
        ref = cref.beam_decode_fullstate(S0[r:r + 1, h:h + 1].contiguous(), _slice(steps, r, h))
        for (go, gd), rr in zip(got[(r, h)], ref):
            assert np.abs(go - rr["o"][0, :, 0]).max() <= tol
            assert np.abs(gd - rr["delta"][0, :, 0]).max() <= tol
