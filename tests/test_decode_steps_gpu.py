"""GPU parity of onela_decode_steps: several decode steps in one call, each
step after the first launched as a programmatic dependent of the step before
it (no handle flag).  Through the C ABI, against the fp64 oracle on the same
seeded inputs: o and every delta record within max-abs 2e-5 (fp32 S0) or
1e-3 (bf16 S0); k records and ancestry rows bit-exact; alpha within a few
fp32 ulps.  The call runs the same kernel as separate onela_decode_step
calls, so it must also agree with them bit for bit.

Covered: the headline workloads at full size, ragged beam counts and tiles
(W not a multiple of 32, W changing from step to step), every split of a
decode into calls (so that a call starts at a depth whose ancestors' keys,
gates and parents come from the record store), calls mixed with single steps
and with folds, a decode deeper than the record store, the bitwise
properties (linearity, relabelled beams, determinism), a captured graph, bad
parents, and a bounded wait running out on purpose."""
import numpy as np
import pytest
import torch

import synth
from tests import _parity as P

pytestmark = pytest.mark.gpu

TC = 2


def run_named(name, chunks, s0_dtype=None, flags=0):
    wl = synth.workload(name)
    if s0_dtype:
        wl = wl.replace(s0_dtype=s0_dtype)
    S0 = P.prompt_state(wl)
    steps = synth.draw_decode(wl)
    gpu, kind = P.run_gpu(S0, steps, wl.qkv_dtype, TC, flags=flags, chunks=chunks(wl.T))
    assert kind == TC
    return P.compare(gpu, P.oracle(S0, steps), steps, wl.s0_dtype)


@pytest.mark.parametrize("name", ["long5k", "long5k_bf16", "op1k"])
def test_whole_decode_in_one_call(name):
    run_named(name, lambda T: [T])


@pytest.mark.parametrize("chunks", [[3, 4], [1, 6], [2, 2, 3], [5, 1, 1], [4, 3]])
def test_decode_split_into_calls(chunks):
    """Launches that start at depth > 1 read the earlier depths' keys, gates,
    parents and deltas from the record store."""
    run_named("long5k", lambda T: chunks)


@pytest.mark.parametrize("name", ["wsweep64", "wsweep128", "wsweep256"])
def test_beam_width_sweep_in_one_call(name):
    run_named(name, lambda T: [T])


def test_tiny_bf16_qkv():
    wl = synth.workload("tiny").replace(qkv_dtype="bf16")
    S0 = synth.draw_s0_direct(wl)
    steps = synth.draw_decode(wl)
    for s0_dtype in ("f32", "bf16"):
        S0c = synth.cast_state(S0, s0_dtype)
        gpu, _ = P.run_gpu(S0c, steps, "bf16", TC, chunks=[wl.T])
        P.compare(gpu, P.oracle(S0c, steps), steps, s0_dtype)


@pytest.mark.parametrize("d,Ws,R,H,chunks", [
    (64, (5, 7, 33, 17), 2, 3, [4]),
    (64, (40, 64, 9, 65, 256), 1, 2, [2, 3]),
    (128, (9, 130, 129, 7), 3, 2, [4]),
    (128, (1, 1, 1, 1), 1, 2, [4]),
    (128, (256, 31, 256, 200, 33, 96), 1, 2, [6]),
    (128, (17, 250, 3), 2, 1, [1, 2]),
])
def test_ragged_shapes(d, Ws, R, H, chunks):
    """Beam counts that change from step to step and leave short or empty
    tiles in the cluster."""
    wl, S0, steps = P.custom_steps(len(Ws) + d + 7, R, H, d, d, Ws, parents="mixed" if R > 1 else "zipf")
    for s0_dtype in ("f32", "bf16"):
        S0c = synth.cast_state(S0, s0_dtype)
        gpu, _ = P.run_gpu(S0c, steps, "bf16", TC, T_max=len(Ws) + 2, W_max=max(Ws) + 3, chunks=chunks)
        P.compare(gpu, P.oracle(S0c, steps), steps, s0_dtype)


def _fixed(kind):
    def f(t, Wp, W, R):
        if kind == "zeros":
            return np.zeros((R, W))
        if kind == "identity":
            return np.tile(np.arange(W) % Wp, (R, 1))
        if kind == "reverse":
            return np.tile((Wp - 1 - np.arange(W)) % Wp, (R, 1))
        return np.full((R, W), (3 * t) % Wp)
    return f


@pytest.mark.parametrize("kind", ["zeros", "identity", "reverse", "lineage"])
def test_adversarial_parents(kind):
    wl, S0, steps = P.custom_steps(11, 1, 2, 128, 128, (64, 200, 256, 256, 256), fixed=_fixed(kind))
    S0c = synth.cast_state(S0, "f32")
    gpu, _ = P.run_gpu(S0c, steps, "bf16", TC, chunks=[5])
    P.compare(gpu, P.oracle(S0c, steps), steps, "f32")


def test_deep_decode_in_one_call():
    """16 steps in one launch (every chain up to 15 ancestors long)."""
    wl, S0, steps = P.custom_steps(12, 1, 2, 64, 64, (16,) * 16)
    S0c = synth.cast_state(S0, "f32")
    gpu, _ = P.run_gpu(S0c, steps, "bf16", TC, chunks=[16])
    P.compare(gpu, P.oracle(S0c, steps), steps, "f32")


@pytest.mark.parametrize("name", ["long5k", "op1k"])
def test_matches_separate_calls_bitwise(name):
    """The same kernel on the same inputs as separate ordinary
    onela_decode_step calls: every output and record bit for bit."""
    wl = synth.workload(name)
    S0 = P.prompt_state(wl)
    steps = synth.draw_decode(wl)
    a, _ = P.run_gpu(S0, steps, "bf16", TC, chunks=[wl.T])
    b, _ = P.run_gpu(S0, steps, "bf16", TC)
    for x, y in zip(a, b):
        for key in ("o", "delta", "alpha", "k", "anc"):
            assert torch.equal(x[key], y[key]), key


def test_identity_gate_keeps_s0():
    """alpha = 1, beta = 0: delta is exactly 0 and o = S0 q for every beam."""
    import linear_attention_beam_shared_b200 as L
    wl, S0, steps = P.custom_steps(13, 1, 2, 128, 128, (32, 96, 96))
    for s in steps:
        s["g"] = torch.zeros_like(s["g"])
        s["beta"] = torch.zeros_like(s["beta"])
    S0c = synth.cast_state(S0, "bf16")
    gpu, _ = P.run_gpu(S0c, steps, "bf16", TC, chunks=[3])
    for g, s in zip(gpu, steps):
        assert float(g["delta"].abs().max()) == 0.0
        ref = torch.einsum("rhij,rbhj->rbhi", S0c.double(), s["q"].double())
        assert float((g["o"].double() - ref).abs().max()) <= P.TOL["bf16"]


def test_linearity_bitwise():
    """Scaling S0 and v by 2 scales o and every delta by exactly 2."""
    wl, S0, steps = P.custom_steps(14, 1, 2, 128, 128, (40, 200, 256))
    S0c = synth.cast_state(S0, "f32")
    a, _ = P.run_gpu(S0c, steps, "bf16", TC, chunks=[3])
    steps2 = [dict(s, v=(s["v"].float() * 2).to(s["v"].dtype)) for s in steps]
    b, _ = P.run_gpu(S0c * 2, steps2, "bf16", TC, chunks=[3])
    for x, y in zip(a, b):
        assert torch.equal(x["o"] * 2, y["o"]) and torch.equal(x["delta"] * 2, y["delta"])


def test_deterministic():
    wl = synth.workload("op1k")
    S0 = P.prompt_state(wl)
    steps = synth.draw_decode(wl)
    a, _ = P.run_gpu(S0, steps, "bf16", TC, chunks=[wl.T])
    b, _ = P.run_gpu(S0, steps, "bf16", TC, chunks=[wl.T])
    for x, y in zip(a, b):
        assert torch.equal(x["o"], y["o"]) and torch.equal(x["delta"], y["delta"])


def test_relabelled_beams_permute_the_outputs():
    """Relabelling the beams of step 2 (and remapping step 3's parents)
    permutes step 2's outputs and leaves step 3's unchanged.  The relabelling
    keeps every beam's tile position parity and position in its tile's
    half-warp pairs, so the arithmetic per beam is the same, bit for bit."""
    wl, S0, steps = P.custom_steps(15, 1, 2, 128, 128, (64, 128, 128))
    S0c = synth.cast_state(S0, "f32")
    a, _ = P.run_gpu(S0c, steps, "bf16", TC, chunks=[3])
    W = 128
    perm = np.arange(W)
    perm = perm.reshape(-1, 2)[np.random.default_rng(3).permutation(W // 2)].reshape(-1)  # keeps parity
    inv = np.argsort(perm)
    s2 = dict(steps[1])
    for key in ("q", "k", "v", "g", "beta", "parents"):
        s2[key] = steps[1][key][:, perm].contiguous()
    s3 = dict(steps[2])
    s3["parents"] = torch.from_numpy(inv[steps[2]["parents"].numpy()].astype(np.int32))
    b, _ = P.run_gpu(S0c, [steps[0], s2, s3], "bf16", TC, chunks=[3])
    assert torch.equal(b[1]["o"], a[1]["o"][:, perm])
    assert torch.equal(b[1]["delta"], a[1]["delta"][:, perm])
    assert torch.equal(b[2]["o"], a[2]["o"])


def test_graph_replay_matches_eager():
    import linear_attention_beam_shared_b200 as L
    wl = synth.workload("long5k")
    S0 = P.prompt_state(wl)
    steps = P.to_dev(synth.draw_decode(wl))
    dec = L.BeamDecoder(wl.R, wl.H, wl.d_k, wl.d_v, wl.W, wl.T, "f32", "bf16", kernel=TC)
    try:
        dec.set_prompt_state(S0.cuda())
        outs = [torch.empty((wl.R, s["W"], wl.H, wl.d_v), device="cuda") for s in steps]
        dec.steps(steps, outs)
        eager = [o.clone() for o in outs]
        dec.reset()
        s = torch.cuda.Stream()
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=s):
            dec.steps(steps, outs, stream=s)
        for _ in range(2):
            dec.reset()
            for o in outs:
                o.fill_(float("nan"))
            g.replay()
            torch.cuda.synchronize()
            for o, e in zip(outs, eager):
                assert torch.equal(o, e)
        del g
        assert dec.status() == 0
    finally:
        dec.close()


def test_bad_parent_is_reported():
    import linear_attention_beam_shared_b200 as L
    wl, S0, steps = P.custom_steps(16, 1, 2, 128, 128, (32, 64, 64))
    steps[2]["parents"] = steps[2]["parents"].clone()
    steps[2]["parents"][0, 5] = 64       # outside [0, W_prev)
    dec = L.BeamDecoder(1, 2, 128, 128, 64, 3, "f32", "bf16", kernel=TC)
    try:
        dec.set_prompt_state(synth.cast_state(S0, "f32").cuda())
        dec.steps(P.to_dev(steps))
        rc, word = L.onela_status_code(dec.h)
        assert rc == L.ONELA_ERR_PARENT and word & 1
    finally:
        dec.close()


def test_bounded_waits_run_out_and_report():
    """The beam warps' wait for the ancestry warp made to expect an arrival
    that never comes: every such wait ends at its 1 ms bound, the kernels
    finish, and the handle reports ONELA_ERR_TIMEOUT (bit 1).  Afterwards,
    with normal waits, the same handle decodes correctly again."""
    import linear_attention_beam_shared_b200 as L
    wl = synth.workload("op1k")
    S0 = P.prompt_state(wl)
    steps = synth.draw_decode(wl)
    ds = P.to_dev(steps)
    dec = L.BeamDecoder(wl.R, wl.H, wl.d_k, wl.d_v, wl.W, wl.T, "f32", "bf16", kernel=TC)
    try:
        dec.set_prompt_state(S0.cuda())
        L.onela_set_wait_policy(dec.h, 1_000_000, stall=True)
        dec.steps(ds)
        rc, word = L.onela_status_code(dec.h)
        assert rc == L.ONELA_ERR_TIMEOUT and word & 2
        L.onela_set_wait_policy(dec.h, 2_000_000_000, stall=False)
        dec.reset()
        outs = dec.steps(ds)
        assert dec.status() == 0
        ref = P.oracle(S0, steps)
        for o, r in zip(outs, ref):
            assert float(np.abs(o.cpu().double().numpy() - r["o"]).max()) <= P.TOL["f32"]
    finally:
        dec.close()


def test_calls_between_folds():
    """Two requests with different bottlenecks; the steps between folds in
    one call each (so later launches replay from a folded state), against
    the unfolded oracle."""
    from oracle import gdn
    from tests import test_fold_gpu as F
    wl, S0, steps = P.custom_steps(31, R=2, H=3, dk=128, dv=128, Ws=[40, 70, 33, 64, 50, 45, 70, 36],
                                   parents="uniform")
    steps = F.narrow(steps, 1, [5, 0])
    steps = F.narrow(steps, 3, [7, 30])
    steps = F.narrow(steps, 4, [2, 2])
    folds = {3: [1, 8], 5: 8, 6: 4}
    S0t = synth.cast_state(S0, "f32")
    gpu, info, used = F.run_with_folds(S0t, steps, "bf16", TC, folds, chunked=True)
    want = F.expected_depths(steps, folds)
    for t, D, S in info:
        assert D.tolist() == want[t].tolist(), (t, D, want[t])
        F.check_state(S, gdn.fold_state(S0t, steps[:t], want[t]))
    P.compare(gpu, P.oracle(S0t, steps), steps, "f32")


def test_deeper_than_the_record_store_in_calls():
    """A store of T_max = 6 depths and a 26-step decode in calls of 4 steps
    (a fold after each), so the records wrap around the store between and
    within launches."""
    from tests import test_fold_gpu as F
    T, TM = 26, 6
    Ws = [12, 20, 16, 20, 24, 16, 20, 12] * 3 + [16, 20]
    wl, S0, steps = P.custom_steps(40, R=2, H=2, dk=128, dv=128, Ws=Ws, parents="uniform")
    for at in range(3, T - 1, 4):
        steps = F.narrow(steps, at, [at % 5, (at + 2) % 7])
    folds = {at + 1: T for at in range(3, T - 1, 4)}
    S0t = synth.cast_state(S0, "f32")
    gpu, info, used = F.run_with_folds(S0t, steps, "bf16", TC, folds, T_max=TM, chunked=True)
    for t, D, _ in info:
        assert D.tolist() == [t - 1, t - 1]
    ref = P.oracle(S0t, steps)
    for t, (g, r) in enumerate(zip(gpu, ref), start=1):
        err = float(np.abs(g["o"].double().numpy() - r["o"]).max())
        assert err <= P.TOL["f32"], (t, err)
        if "delta" in g:
            err = float(np.abs(g["delta"].double().numpy() - r["delta"]).max())
            assert err <= P.TOL["f32"], (t, err)
            assert torch.equal(g["k"], steps[t - 1]["k"])
