"""GPU parity of the beam selection (onela_select_beams, through the C ABI)
against the oracle (oracle/beam.py): parent, token and score bit-exact, on
seeded inputs with ties, -inf and NaN, from a single chunk of candidates to
several merge rounds."""
import numpy as np
import pytest
import torch

from oracle import beam

pytestmark = pytest.mark.gpu


def draw(R, W_prev, C, seed, ties=False, specials=False):
    rng = np.random.default_rng(seed)
    if ties:
        bs = rng.integers(-4, 1, (R, W_prev)).astype(np.float32)
        lp = -rng.integers(0, 8, (R, W_prev, C)).astype(np.float32) * 0.5
    else:
        bs = (-rng.exponential(3.0, (R, W_prev))).astype(np.float32)
        lp = np.log(rng.dirichlet(np.ones(C), (R, W_prev))).astype(np.float32)
    if specials:
        m = rng.random(lp.shape)
        lp[m < 0.05] = -np.inf
        lp[(m >= 0.05) & (m < 0.07)] = np.nan
    return bs, lp


def run_gpu(bs, lp, W):
    import linear_attention_beam_shared_b200 as L
    p, t, s = L.onela_select_beams(torch.from_numpy(bs).cuda(), torch.from_numpy(lp).cuda(), W)
    torch.cuda.synchronize()
    return p.cpu().numpy(), t.cpu().numpy(), s.cpu().numpy()


def check(bs, lp, W):
    p, t, s = run_gpu(bs, lp, W)
    rp, rt, rs = beam.select_beams(bs, lp, W)
    np.testing.assert_array_equal(p, rp)
    np.testing.assert_array_equal(t, rt)
    # bit-exact, NaN included
    np.testing.assert_array_equal(s.view(np.uint32), rs.view(np.uint32))


@pytest.mark.parametrize("R,W_prev,C,W", [
    (1, 1, 1, 1), (1, 8, 8, 8), (3, 16, 32, 16), (2, 50, 101, 50),      # one chunk, ragged
    (1, 256, 256, 256), (4, 256, 256, 256),                              # the headline beam set
    (2, 1024, 256, 1024), (1, 512, 40, 2048), (1, 3, 3000, 7),           # merge rounds, W = 2048
])
@pytest.mark.parametrize("kind", ["smooth", "ties", "specials"])
def test_select_matches_oracle(R, W_prev, C, W, kind):
    bs, lp = draw(R, W_prev, C, seed=R * 1000 + W_prev + C + W, ties=kind == "ties", specials=kind == "specials")
    check(bs, lp, W)


def test_select_every_candidate():
    bs, lp = draw(2, 30, 40, seed=5, ties=True)
    check(bs, lp, 1200)


def test_select_feeds_the_decode():
    """The selected parents drive a decode step directly on the device."""
    import linear_attention_beam_shared_b200 as L
    import synth
    from tests import _parity as P
    wl = synth.workload("tiny")
    S0 = P.prompt_state(wl)
    steps = synth.draw_decode(wl)
    bs, lp = draw(wl.R, 1, 8, seed=9)   # step 1: one root, 8 children
    parent, _, _ = L.onela_select_beams(torch.from_numpy(bs).cuda(), torch.from_numpy(lp).cuda(), wl.W)
    assert bool((parent == 0).all())
    st = steps[0]
    st["parents"] = parent.cpu()
    gpu, _ = P.run_gpu(S0, [st], wl.qkv_dtype, L.ONELA_KERNEL_SIMT)
    P.compare(gpu, P.oracle(S0, [st]), [st], wl.s0_dtype)
