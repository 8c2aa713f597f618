"""GPU parity of the folding extension (onela_fold, through the C ABI): the
folded depth, the folded root state and every output of a decode that folds
on the way, against the fp64 oracle.

The extension addresses the replay cost that grows with decode depth (the
evolve.pub review's Summary and Weaknesses).  Beam trees get bottlenecks (a
step whose beams are all children of one beam), so that later beams share
an ancestor prefix.

Tolerances: with an fp32 state the fold adds the fp32 rounding of a few
multiply-adds per element, far below the decode's own 2e-5, so the outputs
are held to the unfolded oracle at the decode's tolerance and the folded
state to 1e-5 of its scale.  A bf16 state is rounded once more when folded:
the folded state must be the oracle's ancestor state rounded to bf16 (one
unit apart at most, where the fp32 result sits next to a rounding
boundary), and the later outputs are held to the oracle's decode continued
from that rounded state, at the bf16 tolerance.
"""
import numpy as np
import pytest
import torch

import synth
from oracle import gdn
from tests import _parity as P

pytestmark = pytest.mark.gpu

REL_TOL_STATE = 1e-5


def narrow(steps, at, beam):
    """Every beam of step `at` (0-based) becomes a child of beam `beam` (per
    request: a list)."""
    s = steps[at]
    par = s["parents"].clone()
    for r, b in enumerate(beam):
        par[r] = min(b, s["W_prev"] - 1)
    s["parents"] = par
    return steps


def run_with_folds(S0, steps, qkv, kernel, folds, flags=0, T_max=None, chunked=False):
    """Decode all steps on the GPU; after step t (1-based) in `folds`, fold
    with max_depth folds[t].  chunked: the steps between two folds go in one
    onela_decode_steps call instead of one onela_decode_step call each.
    Returns per-step outputs, records and ancestry (records only for the
    depths the store still holds, ancestry only while t <= T_max) and, per
    fold, (t, fold depth [R], root state)."""
    import linear_attention_beam_shared_b200 as L
    R, H, dv, dk = S0.shape
    s0_dtype = "bf16" if S0.dtype == torch.bfloat16 else "f32"
    dec = L.BeamDecoder(R, H, dk, dv, max(s["W"] for s in steps), T_max or len(steps), s0_dtype, qkv,
                        kernel=kernel, flags=flags)
    try:
        ds = P.to_dev(steps)
        dec.set_prompt_state(S0.cuda())
        outs, fold_info = [], []
        pending = []
        for t, s in enumerate(ds, start=1):
            if chunked:
                pending.append(s)
                if t not in folds and t < len(ds):
                    continue
                outs += dec.steps(pending)
                pending = []
            else:
                outs.append(dec.step(s["q"], s["k"], s["v"], s["g"], s["beta"], s["parents"]))
            for md in as_list(folds.get(t, [])):
                dec.fold(md)
            if t in folds:
                fold_info.append((t, dec.fold_depth().cpu().numpy(), dec.root_state().cpu()))
        assert dec.status() == 0
        res = []
        T, TM = len(steps), T_max or len(steps)
        for t, o in enumerate(outs, start=1):
            r = {"o": o.cpu()}
            if t > T - TM:
                a, d, kr = dec.records(t)
                r.update({"alpha": a.cpu().permute(0, 2, 1).contiguous(),
                          "delta": d.cpu().permute(0, 2, 1, 3).contiguous(),
                          "k": kr.cpu().permute(0, 2, 1, 3).contiguous()})
            if t <= TM and t > T - TM:
                r["anc"] = dec.ancestry(t).cpu()
            res.append(r)
        return res, fold_info, dec.kernel
    finally:
        dec.close()


def as_list(x):
    return list(x) if isinstance(x, (list, tuple)) else [x]


def expected_depths(steps, folds):
    """The oracle's fold depth after the folds of each step (never below the
    previous)."""
    out, prev = {}, None
    for t, mds in sorted(folds.items()):
        for md in as_list(mds):
            D, _ = gdn.common_ancestor_depth([s["parents"].numpy() for s in steps[:t]], t, min(md, t))
            if prev is not None:
                D = np.maximum(D, prev)
            prev = D
        out[t] = prev
    return out


def check_state(S_gpu, S_ref):
    scale = max(1.0, float(np.abs(S_ref).max()))
    err = float(np.abs(S_gpu.double().numpy() - S_ref).max())
    assert err <= REL_TOL_STATE * scale, (err, scale)


def kernel_id(kind):
    import linear_attention_beam_shared_b200 as L
    return {"simt": L.ONELA_KERNEL_SIMT, "tc": L.ONELA_KERNEL_TC}[kind]


@pytest.mark.parametrize("kind", ["simt", "tc"])
@pytest.mark.parametrize("pdl", [0, 1])
def test_fold_fp32_state_matches_the_unfolded_decode(kind, pdl):
    """Two requests with different bottlenecks, folds after steps 3 (twice in
    a row: to depth 1, then as deep as shared), 5 and 6 (limited to depth 4):
    folded depths, folded states and all outputs, records and ancestry rows
    against the unfolded oracle."""
    import linear_attention_beam_shared_b200 as L
    dk = dv = 128 if kind == "tc" else 48
    wl, S0, steps = P.custom_steps(31, R=2, H=3, dk=dk, dv=dv, Ws=[40, 70, 33, 64, 50, 45, 70, 36],
                                   parents="uniform")
    steps = narrow(steps, 1, [5, 0])     # step 2: request 0 under beam 5, request 1 under beam 0
    steps = narrow(steps, 3, [7, 30])    # step 4
    steps = narrow(steps, 4, [2, 2])     # step 5
    folds = {3: [1, 8], 5: 8, 6: 4}
    S0t = synth.cast_state(S0, "f32")
    flags = L.ONELA_FLAG_PDL if pdl else 0
    gpu, info, used = run_with_folds(S0t, steps, "bf16", kernel_id(kind), folds, flags=flags)
    assert used == kernel_id(kind)
    want = expected_depths(steps, folds)
    for t, D, S in info:
        assert D.tolist() == want[t].tolist(), (t, D, want[t])
        check_state(S, gdn.fold_state(S0t, steps[:t], want[t]))
    assert want[6].min() >= 3   # the test reaches deep folds
    ref = P.oracle(S0t, steps)
    P.compare(gpu, ref, steps, "f32")


@pytest.mark.parametrize("kind", ["simt", "tc"])
def test_fold_bf16_state(kind):
    """A bf16 state: the folded state is the oracle's ancestor state rounded
    once; later outputs follow the oracle's decode from that rounded state."""
    dk = dv = 128 if kind == "tc" else 64
    wl, S0, steps = P.custom_steps(32, R=2, H=2, dk=dk, dv=dv, Ws=[16, 40, 24, 40, 30, 20], parents="uniform")
    steps = narrow(steps, 2, [3, 9])     # step 3: shared depth 2 for later beams
    S0t = synth.cast_state(S0, "bf16")
    t_f = 4
    gpu, info, _ = run_with_folds(S0t, steps, "bf16", kernel_id(kind), {t_f: t_f})
    (_, D, S), = info
    want = expected_depths(steps, {t_f: t_f})[t_f]
    assert D.tolist() == want.tolist() and (D >= 2).all()
    Sf = gdn.fold_state(S0t, steps[:t_f], D)
    ref16 = synth.cast_state(Sf, "bf16")
    diff = (S.float() - ref16.float()).abs()
    ulp = torch.maximum(S.float().abs(), ref16.float().abs()) * 2.0 ** -7
    assert bool((diff <= ulp + 1e-6).all())
    assert float((diff > 0).float().mean()) < 0.01
    # steps up to the fold: the unfolded oracle
    full = P.oracle(S0t, steps)
    for t in range(t_f):
        assert float(np.abs(gpu[t]["o"].double().numpy() - full[t]["o"]).max()) <= P.TOL["bf16"]
    # later steps: per request, the oracle continued from the rounded folded state
    for r in range(S0.shape[0]):
        d = int(D[r])
        sub = [{k: (v[r:r + 1] if isinstance(v, torch.Tensor) else v) for k, v in s.items()} for s in steps]
        W_d = sub[d - 1]["parents"].shape[1]
        S_prev = np.repeat(gdn.to_f64(ref16[r:r + 1])[:, None], W_d, axis=1)
        cont = gdn.beam_decode_fullstate(S0t[r:r + 1], sub[d:], S_prev=S_prev)
        for t in range(t_f, len(steps)):
            err = float(np.abs(gpu[t]["o"][r:r + 1].double().numpy() - cont[t - d]["o"]).max())
            assert err <= P.TOL["bf16"], (r, t + 1, err)


@pytest.mark.parametrize("kind", ["simt", "tc"])
@pytest.mark.parametrize("pdl", [0, 1])
def test_fold_every_step_of_a_single_beam(kind, pdl):
    """W = 1 at every step, folded to full depth after each: every later step
    replays nothing (its parent is the folded state), and the outputs are
    the sequential GDN recurrence's."""
    import linear_attention_beam_shared_b200 as L
    dk = dv = 128 if kind == "tc" else 32
    T = 9
    wl, S0, steps = P.custom_steps(33, R=2, H=2, dk=dk, dv=dv, Ws=[1] * T, parents="uniform")
    S0t = synth.cast_state(S0, "f32")
    folds = {t: T for t in range(1, T)}
    gpu, info, _ = run_with_folds(S0t, steps, "bf16", kernel_id(kind), folds,
                                  flags=L.ONELA_FLAG_PDL if pdl else 0)
    for t, D, _ in info:
        assert D.tolist() == [t, t]
    P.compare(gpu, P.oracle(S0t, steps), steps, "f32")


@pytest.mark.parametrize("kind", ["simt", "tc"])
def test_fold_without_a_shared_ancestor_changes_nothing(kind):
    """Beams that split at the root: the fold depth stays 0, the root state is
    the prompt state and the decode is the unfolded one."""
    dk = dv = 128 if kind == "tc" else 40
    wl, S0, steps = P.custom_steps(34, R=1, H=2, dk=dk, dv=dv, Ws=[8, 8, 8, 8], parents="uniform")
    steps[1]["parents"] = torch.arange(8, dtype=torch.int32)[None]
    steps[2]["parents"] = torch.arange(8, dtype=torch.int32)[None]
    S0t = synth.cast_state(S0, "f32")
    gpu, info, _ = run_with_folds(S0t, steps, "bf16", kernel_id(kind), {2: 2, 3: 3})
    for _, D, S in info:
        assert D.tolist() == [0]
        assert torch.equal(S, S0t)
    P.compare(gpu, P.oracle(S0t, steps), steps, "f32")


@pytest.mark.parametrize("kind", ["simt", "tc"])
def test_reset_after_a_fold_returns_to_the_prompt_state(kind):
    import linear_attention_beam_shared_b200 as L
    dk = dv = 128 if kind == "tc" else 64
    wl, S0, steps = P.custom_steps(35, R=1, H=2, dk=dk, dv=dv, Ws=[8, 12, 8], parents="uniform")
    steps = narrow(steps, 1, [3])
    S0t = synth.cast_state(S0, "f32")
    dec = L.BeamDecoder(1, 2, dk, dv, 12, 3, "f32", "bf16", kernel=kernel_id(kind))
    try:
        ds = P.to_dev(steps)
        dec.set_prompt_state(S0t.cuda())
        for s in ds[:2]:
            dec.step(s["q"], s["k"], s["v"], s["g"], s["beta"], s["parents"])
        dec.fold()
        assert dec.fold_depth().cpu().tolist() == [1]
        assert not torch.equal(dec.root_state().cpu(), S0t)
        dec.reset()
        assert dec.fold_depth().cpu().tolist() == [0]
        assert torch.equal(dec.root_state().cpu(), S0t)
        assert torch.equal(dec.prompt_state().cpu(), S0t)
        outs = [dec.step(s["q"], s["k"], s["v"], s["g"], s["beta"], s["parents"]).cpu() for s in ds]
        assert dec.status() == 0
    finally:
        dec.close()
    ref = P.oracle(S0t, steps)
    for o, r in zip(outs, ref):
        assert float(np.abs(o.double().numpy() - r["o"]).max()) <= P.TOL["f32"]


def test_fold_before_any_step_and_depth_zero_are_no_ops():
    import linear_attention_beam_shared_b200 as L
    wl, S0, steps = P.custom_steps(36, R=1, H=1, dk=32, dv=32, Ws=[4, 4], parents="uniform")
    S0t = synth.cast_state(S0, "f32")
    dec = L.BeamDecoder(1, 1, 32, 32, 4, 2, "f32", "f32", kernel=L.ONELA_KERNEL_SIMT)
    try:
        with pytest.raises(L.OnelaError):
            dec.fold(1)                      # no prompt state yet
        dec.set_prompt_state(S0t.cuda())
        dec.fold(1)
        assert dec.fold_depth().cpu().tolist() == [0]
        with pytest.raises(L.OnelaError):
            L.onela_fold(dec.h, -1)
        s = P.to_dev(steps)[0]
        dec.step(s["q"].float(), s["k"].float(), s["v"].float(), s["g"], s["beta"], s["parents"])
        dec.fold(0)
        assert dec.fold_depth().cpu().tolist() == [0]
        assert dec.status() == 0
    finally:
        dec.close()


@pytest.mark.parametrize("name", ["long5k"])
def test_fold_full_size(name):
    """The full workload (16 heads, d = 128, 256 beams, 7 steps, fp32 state
    from the prompt): all beams of step 3 under one beam, a fold after step 4
    (depth 2 shared), steps 5-7 against the unfolded oracle."""
    wl = synth.workload(name)
    S0t = P.prompt_state(wl)
    steps = synth.draw_decode(wl)
    steps = narrow(steps, 2, [11] * wl.R)
    gpu, info, _ = run_with_folds(S0t, steps, wl.qkv_dtype, 1, {4: 4})
    (_, D, S), = info
    want = expected_depths(steps, {4: 4})[4]
    assert D.tolist() == want.tolist() and (D >= 2).all()
    check_state(S, gdn.fold_state(S0t, steps[:4], want))
    P.compare(gpu, P.oracle(S0t, steps), steps, wl.s0_dtype)


@pytest.mark.parametrize("kind", ["simt", "tc"])
@pytest.mark.parametrize("pdl", [0, 1])
def test_decode_deeper_than_the_record_store(kind, pdl):
    """A store of T_max = 6 depths and a 26-step decode: every beam of steps
    4, 8, ..., 24 is a child of one beam and a fold follows each of them, so
    no step replays more than 5 depths while the records wrap around the
    store.  Every output, and the delta records the store still holds,
    against the fp64 oracle of the whole 26-step tree."""
    import linear_attention_beam_shared_b200 as L
    T, TM = 26, 6
    dk = dv = 128 if kind == "tc" else 32
    Ws = [12, 20, 16, 20, 24, 16, 20, 12] * 3 + [16, 20]
    wl, S0, steps = P.custom_steps(40, R=2, H=2, dk=dk, dv=dv, Ws=Ws, parents="uniform")
    for at in range(3, T - 1, 4):
        steps = narrow(steps, at, [at % 5, (at + 2) % 7])
    folds = {at + 1: T for at in range(3, T - 1, 4)}
    S0t = synth.cast_state(S0, "f32")
    gpu, info, used = run_with_folds(S0t, steps, "bf16", kernel_id(kind), folds,
                                     flags=L.ONELA_FLAG_PDL if pdl else 0, T_max=TM)
    assert used == kernel_id(kind)
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


@pytest.mark.parametrize("TM", [5, 6, 8])
@pytest.mark.parametrize("pdl", [0, 1])
def test_step_after_a_fold_lags_or_waits(TM, pdl):
    """The tensor-core step right after a fold replays from the folded state
    before that fold while its depths still fit the record store, and waits
    for the fold otherwise.  With a fold after every fourth step (steps
    4k replay 4 depths, so the store needs at least 5), the step after the
    fold at 4k replays 5 depths from the fold before (4 after the first
    fold): a 5-depth store takes that only after the first fold and waits
    after the others, 6 and 8 never wait.  Outputs of every step and the
    folded depths against the fp64 oracle."""
    import linear_attention_beam_shared_b200 as L
    T = 18
    Ws = [8, 24, 16, 20, 12, 24, 16, 8, 20] * 2
    wl, S0, steps = P.custom_steps(47 + TM, R=2, H=3, dk=64, dv=64, Ws=Ws, parents="zipf")
    for at in range(3, T - 1, 4):
        steps = narrow(steps, at, [at % 3, (at + 1) % 5])
    folds = {at + 1: T for at in range(3, T - 1, 4)}
    S0t = synth.cast_state(S0, "f32")
    gpu, info, used = run_with_folds(S0t, steps, "bf16", kernel_id("tc"), folds,
                                     flags=L.ONELA_FLAG_PDL if pdl else 0, T_max=TM)
    assert used == kernel_id("tc")
    for t, D, _ in info:
        assert D.tolist() == [t - 1, t - 1]
    ref = P.oracle(S0t, steps)
    for t, (g, r) in enumerate(zip(gpu, ref), start=1):
        err = float(np.abs(g["o"].double().numpy() - r["o"]).max())
        assert err <= P.TOL["f32"], (t, err)


def test_fold_tc_store_of_20_depths():
    """A tensor-core handle whose record store is deeper than the one-launch
    fold serves (20 depths): folds take the general path, then the folded
    state's operand image; a 40-step decode through it against the oracle."""
    import linear_attention_beam_shared_b200 as L
    T, TM = 40, 20
    Ws = [16, 24, 20, 12, 24, 16, 20, 28] * 5
    wl, S0, steps = P.custom_steps(52, R=1, H=2, dk=128, dv=128, Ws=Ws, parents="uniform")
    for at in range(9, T - 1, 10):
        steps = narrow(steps, at, [at % 7])
    folds = {at + 1: T for at in range(9, T - 1, 10)}
    S0t = synth.cast_state(S0, "f32")
    gpu, info, used = run_with_folds(S0t, steps, "bf16", kernel_id("tc"), folds, flags=L.ONELA_FLAG_PDL, T_max=TM)
    assert used == kernel_id("tc")
    for t, D, _ in info:
        assert D.tolist() == [t - 1]
    ref = P.oracle(S0t, steps)
    for t, (g, r) in enumerate(zip(gpu, ref), start=1):
        assert float(np.abs(g["o"].double().numpy() - r["o"]).max()) <= P.TOL["f32"], t


@pytest.mark.parametrize("kind", ["simt", "tc"])
def test_unfolded_window_overflow_is_reported(kind):
    """With nothing shared to fold, a decode that goes past T_max unfolded
    depths is stopped: the host refuses step T_max + 1 without a fold, and
    after a fold that folded nothing the device reports the overflow
    (ONELA_ERR_CAPACITY) instead of replaying overwritten records.  Records
    of depths that left the store cannot be read back."""
    import linear_attention_beam_shared_b200 as L
    TM = 4
    dk = dv = 128 if kind == "tc" else 32
    wl, S0, steps = P.custom_steps(41, R=1, H=2, dk=dk, dv=dv, Ws=[8] * 6, parents="uniform")
    for t in range(1, 6):
        steps[t]["parents"] = torch.arange(8, dtype=torch.int32)[None]
    dec = L.BeamDecoder(1, 2, dk, dv, 8, TM, "f32", "bf16", kernel=kernel_id(kind))
    try:
        ds = P.to_dev(steps)
        dec.set_prompt_state(synth.cast_state(S0, "f32").cuda())
        for s in ds[:TM]:
            dec.step(s["q"], s["k"], s["v"], s["g"], s["beta"], s["parents"])
        s = ds[TM]
        with pytest.raises(L.OnelaError) as e:
            dec.step(s["q"], s["k"], s["v"], s["g"], s["beta"], s["parents"])
        assert e.value.code == L.ONELA_ERR_CAPACITY
        dec.fold()
        assert dec.fold_depth().cpu().tolist() == [0]
        dec.step(s["q"], s["k"], s["v"], s["g"], s["beta"], s["parents"])
        with pytest.raises(L.OnelaError) as e:
            dec.status()
        assert e.value.code == L.ONELA_ERR_CAPACITY
        with pytest.raises(L.OnelaError):
            L.onela_read_records(dec.h, 1, 8)
        dec.reset()
        assert dec.status() == 0
    finally:
        dec.close()


@pytest.mark.parametrize("kind", ["simt", "tc"])
def test_fold_with_more_beams_than_threads(kind):
    """600 beams: the tensor-core fold compares the ancestry rows of beams
    past its 256 threads in a second loop.  Request 0 narrows to one beam at
    step 2, request 1 does not."""
    dk = dv = 128 if kind == "tc" else 32
    wl, S0, steps = P.custom_steps(42, R=2, H=2, dk=dk, dv=dv, Ws=[300, 600, 600, 500], parents="uniform")
    par = steps[1]["parents"].clone()
    par[0] = 17
    par[1] = torch.arange(600, dtype=torch.int32) % 300
    steps[1]["parents"] = par
    S0t = synth.cast_state(S0, "f32")
    gpu, info, _ = run_with_folds(S0t, steps, "bf16", kernel_id(kind), {3: 3})
    (_, D, S), = info
    want = expected_depths(steps, {3: 3})[3]
    assert D.tolist() == want.tolist() and D.tolist()[0] >= 1
    check_state(S, gdn.fold_state(S0t, steps[:3], want))
    P.compare(gpu, P.oracle(S0t, steps), steps, "f32")


@pytest.mark.parametrize("kind", ["simt", "tc"])
def test_single_beam_decode_through_a_small_store(kind):
    """W = 1 for 20 steps through a 4-depth store, folded after every step
    (each fold takes the step's own depth): the sequential GDN recurrence's
    outputs, while the store wraps five times."""
    T, TM = 20, 4
    dk = dv = 128 if kind == "tc" else 32
    wl, S0, steps = P.custom_steps(43, R=2, H=2, dk=dk, dv=dv, Ws=[1] * T, parents="uniform")
    S0t = synth.cast_state(S0, "f32")
    gpu, info, _ = run_with_folds(S0t, steps, "bf16", kernel_id(kind), {t: T for t in range(1, T)}, T_max=TM)
    for t, D, _ in info:
        assert D.tolist() == [t, t]
    ref = P.oracle(S0t, steps)
    for t, (g, r) in enumerate(zip(gpu, ref), start=1):
        assert float(np.abs(g["o"].double().numpy() - r["o"]).max()) <= P.TOL["f32"], t


def test_fold_tc_d256():
    """Folding on a d = 256 tensor-core handle (the general fold, then the
    folded state's operand image): outputs against the unfolded oracle."""
    import linear_attention_beam_shared_b200 as L
    wl, S0, steps = P.custom_steps(33, R=1, H=2, dk=256, dv=256, Ws=[40, 64, 33, 64, 50], parents="uniform")
    steps = narrow(steps, 1, [5])
    steps = narrow(steps, 3, [7])
    folds = {3: 8, 5: 8}
    S0t = synth.cast_state(S0, "f32")
    gpu, info, used = run_with_folds(S0t, steps, "bf16", L.ONELA_KERNEL_TC, folds)
    assert used == L.ONELA_KERNEL_TC
    want = expected_depths(steps, folds)
    for t, D, S in info:
        assert D.tolist() == want[t].tolist()
        check_state(S, gdn.fold_state(S0t, steps[:t], want[t]))
    P.compare(gpu, P.oracle(S0t, steps), steps, "f32")
