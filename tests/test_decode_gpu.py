"""GPU parity: the CUDA decode path (through the C ABI) against the fp64
oracle on the same seeded inputs.  o and delta within max-abs 2e-5 (fp32 S0)
or 1e-3 (bf16 S0); k records, ancestry rows bit-exact; alpha records within a
few fp32 ulps of exp(g)."""
import numpy as np
import pytest
import torch

import synth
from tests import _parity as P

pytestmark = pytest.mark.gpu


def kernels_for(dk, dv, qkv):
    import linear_attention_beam_shared_b200 as L
    ks = [L.ONELA_KERNEL_SIMT]
    if qkv == "bf16" and dk == dv and dk in (64, 128, 256) and _tc_available():
        ks.append(L.ONELA_KERNEL_TC)
    return ks


def _tc_available():
    import linear_attention_beam_shared_b200 as L
    try:
        h = L.onela_create(1, 1, 128, 128, 8, 2, "f32", "bf16", L.ONELA_KERNEL_TC)
    except L.OnelaError as e:
        if e.code == L.ONELA_ERR_UNSUPPORTED:
            return False
        raise
    L.onela_destroy(h)
    return True


def _all_kernels():
    import linear_attention_beam_shared_b200 as L
    return [L.ONELA_KERNEL_SIMT, L.ONELA_KERNEL_TC]


def _skip_unavailable(kernel, dk, dv, qkv):
    if kernel not in kernels_for(dk, dv, qkv):
        pytest.skip("kernel does not serve this shape")


def run_workload(name, kernel, s0_dtype=None, flags=0, s0_split=0):
    wl = synth.workload(name)
    if s0_dtype:
        wl = wl.replace(s0_dtype=s0_dtype)
    _skip_unavailable(kernel, wl.d_k, wl.d_v, wl.qkv_dtype)
    S0 = P.prompt_state(wl)
    steps = synth.draw_decode(wl)
    gpu, _ = P.run_gpu(S0, steps, wl.qkv_dtype, kernel, flags=flags, s0_split=s0_split)
    ref = P.oracle(S0, steps)
    return P.compare(gpu, ref, steps, wl.s0_dtype)


@pytest.mark.parametrize("name", ["op1k", "long5k", "long5k_bf16"])
def test_tc_with_programmatic_launch(name):
    """Steps 2..T start before the previous step ends (inputs resident)."""
    import linear_attention_beam_shared_b200 as L
    run_workload(name, 2, flags=L.ONELA_FLAG_PDL)


def test_tc_three_term_split():
    run_workload("long5k", 2, s0_split=3)


@pytest.mark.parametrize("kernel", [1, 2])
@pytest.mark.parametrize("s0_dtype", ["f32", "bf16"])
def test_tiny(kernel, s0_dtype):
    run_workload("tiny", kernel, s0_dtype)


@pytest.mark.parametrize("kernel", [1, 2])
def test_op1k(kernel):
    run_workload("op1k", kernel)


@pytest.mark.parametrize("kernel", [1, 2])
@pytest.mark.parametrize("name", ["long5k", "long5k_bf16"])
def test_long5k(kernel, name):
    run_workload(name, kernel)


@pytest.mark.parametrize("kernel", [1, 2])
@pytest.mark.parametrize("d,Ws,R,H,qkv", [
    (64, (5, 7, 33, 17), 2, 3, "bf16"),
    (64, (5, 7, 33, 17), 1, 2, "f32"),
    (96, (3, 40, 40), 1, 2, "bf16"),
    (128, (1, 1, 1, 1), 1, 2, "bf16"),
    (128, (9, 130, 129, 7), 3, 2, "bf16"),
    (256, (20, 19, 21), 1, 2, "bf16"),
    (32, (300, 257, 260), 1, 1, "f32"),
])
def test_ragged_shapes(kernel, d, Ws, R, H, qkv):
    _skip_unavailable(kernel, d, d, qkv)
    wl, S0, steps = P.custom_steps(len(Ws) + d, R, H, d, d, Ws, qkv_dtype=qkv,
                                   parents="mixed" if R > 1 else "zipf")
    for s0_dtype in ("f32", "bf16"):
        S0c = synth.cast_state(S0, s0_dtype)
        gpu, _ = P.run_gpu(S0c, steps, qkv, kernel, T_max=len(Ws) + 2, W_max=max(Ws) + 3)
        P.compare(gpu, P.oracle(S0c, steps), steps, s0_dtype)


def _fixed(kind):
    def f(t, Wp, W, R):
        if kind == "zeros":
            return np.zeros((R, W))
        if kind == "identity":
            return np.tile(np.arange(W) % Wp, (R, 1))
        if kind == "reverse":
            return np.tile((Wp - 1 - np.arange(W)) % Wp, (R, 1))
        return np.full((R, W), (3 * t) % Wp)          # one surviving lineage
    return f


@pytest.mark.parametrize("kernel", [1, 2])
@pytest.mark.parametrize("kind", ["zeros", "identity", "reverse", "lineage"])
def test_adversarial_parents(kernel, kind):
    _skip_unavailable(kernel, 128, 128, "bf16")
    wl, S0, steps = P.custom_steps(7, 2, 2, 128, 128, (64, 64, 64, 64, 64, 64), fixed=_fixed(kind))
    S0c = synth.cast_state(S0, "f32")
    gpu, _ = P.run_gpu(S0c, steps, "bf16", kernel)
    P.compare(gpu, P.oracle(S0c, steps), steps, "f32")


@pytest.mark.parametrize("kernel", [1, 2])
def test_wide_beams_gathered_ancestry(kernel):
    """W_max * T_max too large for the tensor-core kernel's shared-memory
    copy of the ancestor rows: it gathers them row by row instead."""
    _skip_unavailable(kernel, 64, 64, "bf16")
    wl, S0, steps = P.custom_steps(16, 1, 2, 64, 64, (600, 600, 600, 600, 600))
    S0c = synth.cast_state(S0, "f32")
    gpu, _ = P.run_gpu(S0c, steps, "bf16", kernel, T_max=8)
    P.compare(gpu, P.oracle(S0c, steps), steps, "f32")


@pytest.mark.parametrize("kernel", [1, 2])
def test_deep_decode(kernel):
    _skip_unavailable(kernel, 64, 64, "bf16")
    wl, S0, steps = P.custom_steps(8, 1, 2, 64, 64, (24,) * 12)
    S0c = synth.cast_state(S0, "f32")
    gpu, _ = P.run_gpu(S0c, steps, "bf16", kernel)
    P.compare(gpu, P.oracle(S0c, steps), steps, "f32")


@pytest.mark.parametrize("T,W,d,R,H", [(24, 40, 64, 2, 3), (32, 256, 128, 1, 4), (20, 33, 128, 1, 2),
                                        (20, 72, 256, 1, 2)])
def test_tc_store_deeper_than_16(T, W, d, R, H):
    """A record store of up to 32 depths on the tensor-core kernel (one CTA
    per SM past 16 depths at d = 128; at d = 256 the image ring and the
    delta staging over it): every step replays up to T - 1
    ancestors, through both the callers' arrays (one onela_decode_steps
    call) and the record store (one call per step)."""
    import linear_attention_beam_shared_b200 as L
    _skip_unavailable(2, d, d, "bf16")
    wl, S0, steps = P.custom_steps(60 + T, R, H, d, d, (W,) * T, parents="zipf")
    S0c = synth.cast_state(S0, "f32")
    ref = P.oracle(S0c, steps)
    for chunks in (None, [T]):
        gpu, used = P.run_gpu(S0c, steps, "bf16", L.ONELA_KERNEL_TC, chunks=chunks)
        assert used == L.ONELA_KERNEL_TC
        P.compare(gpu, ref, steps, "f32")


@pytest.mark.parametrize("Ws,d,H", [((64, 2048, 1500, 4096), 64, 2), ((2048, 2048, 1111), 128, 1)])
def test_tc_wide_beam_sets(Ws, d, H):
    """Beam sets past 1024 on the tensor-core kernel (up to 4096: 128 beam
    tiles per head, the parents of earlier steps read from global memory once
    they no longer fit the kernel's shared copy), through the callers' arrays
    and through the record store, against the fp64 oracle."""
    import linear_attention_beam_shared_b200 as L
    _skip_unavailable(2, d, d, "bf16")
    wl, S0, steps = P.custom_steps(80 + d, 1, H, d, d, Ws, parents="zipf")
    S0c = synth.cast_state(S0, "f32")
    ref = P.oracle(S0c, steps)
    for chunks in (None, [len(Ws)]):
        gpu, used = P.run_gpu(S0c, steps, "bf16", L.ONELA_KERNEL_TC, chunks=chunks)
        assert used == L.ONELA_KERNEL_TC
        P.compare(gpu, ref, steps, "f32")


@pytest.mark.parametrize("kernel", [1, 2])
def test_identity_gate_keeps_s0(kernel):
    """alpha = 1 (g = 0), beta = 0: delta is exactly zero and o = S0 q."""
    _skip_unavailable(kernel, 128, 128, "bf16")
    wl, S0, steps = P.custom_steps(9, 1, 2, 128, 128, (16, 40, 40))
    for s in steps:
        s["g"].zero_()
        s["beta"].zero_()
    S0c = synth.cast_state(S0, "f32")
    gpu, _ = P.run_gpu(S0c, steps, "bf16", kernel)
    for g, s in zip(gpu, steps):
        assert torch.count_nonzero(g["delta"]) == 0
        assert torch.all(g["alpha"] == 1.0)
        ref = np.einsum("rhij,rwhj->rwhi", S0c.double().numpy(), s["q"].double().numpy())
        assert np.abs(g["o"].double().numpy() - ref).max() <= P.TOL["f32"]


@pytest.mark.parametrize("kernel", [1, 2])
def test_linearity(kernel):
    """o and delta are linear in (S0, v), and both kernels keep it bitwise:
    scaling by 2 is exact in every fp32 operation, in the bf16 terms of the
    S0 image and in the tensor-core products."""
    _skip_unavailable(kernel, 128, 128, "bf16")
    wl, S0, steps = P.custom_steps(10, 1, 2, 128, 128, (8, 33, 33, 20))
    S0c = synth.cast_state(S0, "f32")
    a, _ = P.run_gpu(S0c, steps, "bf16", kernel)
    steps2 = [dict(s, v=(2 * s["v"].float()).to(s["v"].dtype)) for s in steps]
    b, _ = P.run_gpu(2 * S0c, steps2, "bf16", kernel)
    for x, y in zip(a, b):
        assert torch.equal(2 * x["o"], y["o"])
        assert torch.equal(2 * x["delta"], y["delta"])


@pytest.mark.parametrize("kernel", [1, 2])
def test_deterministic(kernel):
    _skip_unavailable(kernel, 128, 128, "bf16")
    wl, S0, steps = P.custom_steps(11, 1, 4, 128, 128, (64, 128, 128))
    S0c = synth.cast_state(S0, "f32")
    a, _ = P.run_gpu(S0c, steps, "bf16", kernel)
    b, _ = P.run_gpu(S0c, steps, "bf16", kernel)
    for x, y in zip(a, b):
        assert torch.equal(x["o"], y["o"]) and torch.equal(x["delta"], y["delta"])


@pytest.mark.parametrize("kernel", [1, 2])
def test_permutation_equivariance(kernel):
    """Relabelling the beams of one step (and remapping the next step's
    parents to the new labels) permutes that step's outputs and delta
    records and leaves every other output unchanged, bit for bit: a beam's
    arithmetic does not depend on its neighbours, its tile or the order in
    which the tile's distinct ancestors are found.  The tensor-core kernel
    visits a beam's element groups in swapped order at odd positions, so
    there the relabelling keeps each beam's parity."""
    import linear_attention_beam_shared_b200 as L
    _skip_unavailable(kernel, 128, 128, "bf16")
    wl, S0, steps = P.custom_steps(13, 2, 2, 128, 128, (40, 70, 70, 50))
    S0c = synth.cast_state(S0, "f32")
    a, _ = P.run_gpu(S0c, steps, "bf16", kernel)
    s = 1                                    # relabel the beams of step 2
    W = steps[s]["W"]
    rng = np.random.default_rng(5)
    if kernel == L.ONELA_KERNEL_TC:
        perm = np.arange(W)
        for par in (0, 1):
            idx = np.arange(par, W, 2)
            perm[idx] = rng.permutation(idx)
    else:
        perm = rng.permutation(W)
    perm = torch.from_numpy(perm)            # new beam i is old beam perm[i]
    inv = torch.empty_like(perm)
    inv[perm] = torch.arange(W)
    steps2 = [dict(x) for x in steps]
    for key in ("q", "k", "v", "g", "beta", "parents"):
        steps2[s][key] = steps[s][key][:, perm].contiguous()
    steps2[s + 1]["parents"] = inv[steps[s + 1]["parents"].long()].to(torch.int32)
    b, _ = P.run_gpu(S0c, steps2, "bf16", kernel)
    assert not torch.equal(perm, torch.arange(W))
    for t, (x, y) in enumerate(zip(a, b)):
        if t == s:
            assert torch.equal(x["o"][:, perm], y["o"])
            assert torch.equal(x["delta"][:, perm], y["delta"])
        else:
            assert torch.equal(x["o"], y["o"]) and torch.equal(x["delta"], y["delta"])


@pytest.mark.parametrize("kernel,flags", [(1, 0), (2, 0), (2, 1)])
def test_graph_replay_matches_eager(kernel, flags):
    import linear_attention_beam_shared_b200 as L
    _skip_unavailable(kernel, 128, 128, "bf16")
    wl, S0, steps = P.custom_steps(12, 1, 4, 128, 128, (32, 96, 96, 96))
    S0c = synth.cast_state(S0, "f32").cuda()
    dsteps = P.to_dev(steps)
    eager, _ = P.run_gpu(S0c.cpu(), steps, "bf16", kernel, read_back=False)
    dec = L.BeamDecoder(1, 4, 128, 128, 96, 4, "f32", "bf16", kernel=kernel, flags=flags)
    try:
        dec.set_prompt_state(S0c)
        outs = [torch.empty((1, s["W"], 4, 128), device="cuda") for s in steps]
        stream = torch.cuda.Stream()
        torch.cuda.synchronize()
        graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(graph, stream=stream):
            for s, o in zip(dsteps, outs):
                dec.step(s["q"], s["k"], s["v"], s["g"], s["beta"], s["parents"], o=o)
        for _ in range(2):
            for o in outs:
                o.zero_()
            graph.replay()
            torch.cuda.synchronize()
            for e, o in zip(eager, outs):
                assert torch.equal(e["o"], o.cpu())
        del graph
    finally:
        dec.close()


def test_bad_parent_is_reported():
    import linear_attention_beam_shared_b200 as L
    wl, S0, steps = P.custom_steps(13, 1, 2, 64, 64, (6, 6, 6))
    steps[1]["parents"][0, 3] = 6          # W_prev is 6: out of range
    dec = L.BeamDecoder(1, 2, 64, 64, 6, 3, "f32", "bf16")
    try:
        dec.set_prompt_state(synth.cast_state(S0, "f32").cuda())
        d = P.to_dev(steps)
        dec.step(d[0]["q"], d[0]["k"], d[0]["v"], d[0]["g"], d[0]["beta"], d[0]["parents"])
        dec.step(d[1]["q"], d[1]["k"], d[1]["v"], d[1]["g"], d[1]["beta"], d[1]["parents"])
        rc, word = L.onela_status_code(dec.h)
        assert rc == L.ONELA_ERR_PARENT and word & 1
        with pytest.raises(L.OnelaError) as ei:
            dec.step(d[2]["q"], d[2]["k"], d[2]["v"], d[2]["g"], d[2]["beta"], d[2]["parents"])
        assert ei.value.code == L.ONELA_ERR_PARENT
        dec.reset()
        assert dec.status() == 0
        dec.step(d[0]["q"], d[0]["k"], d[0]["v"], d[0]["g"], d[0]["beta"], d[0]["parents"])
        assert dec.status() == 0
    finally:
        dec.close()


def test_host_side_errors():
    import linear_attention_beam_shared_b200 as L
    wl, S0, steps = P.custom_steps(14, 1, 2, 64, 64, (4, 4, 4))
    d = P.to_dev(steps)
    dec = L.BeamDecoder(1, 2, 64, 64, 4, 2, "f32", "bf16")
    try:
        s = d[0]
        with pytest.raises(L.OnelaError) as ei:
            dec.step(s["q"], s["k"], s["v"], s["g"], s["beta"], s["parents"])
        assert ei.value.code == L.ONELA_ERR_STATE
        dec.set_prompt_state(synth.cast_state(S0, "f32").cuda())
        o = torch.empty((1, 4, 2, 64), device="cuda")
        with pytest.raises(L.OnelaError) as ei:        # W_prev must be 1 at step 1
            L.onela_decode_step(dec.h, 4, 4, s["q"], s["k"], s["v"], s["g"], s["beta"], s["parents"], o)
        assert ei.value.code == L.ONELA_ERR_ARG
        dec.step(s["q"], s["k"], s["v"], s["g"], s["beta"], s["parents"])
        dec.step(d[1]["q"], d[1]["k"], d[1]["v"], d[1]["g"], d[1]["beta"], d[1]["parents"])
        with pytest.raises(L.OnelaError) as ei:        # T_max = 2
            dec.step(d[2]["q"], d[2]["k"], d[2]["v"], d[2]["g"], d[2]["beta"], d[2]["parents"])
        assert ei.value.code == L.ONELA_ERR_CAPACITY
        dec.reset()
        if dec.kernel == L.ONELA_KERNEL_TC:    # 16-byte aligned tiles
            o_off = torch.empty(1 * 4 * 2 * 64 + 1, device="cuda")[1:].view(1, 4, 2, 64)
            with pytest.raises(L.OnelaError) as ei:
                L.onela_decode_step(dec.h, 1, 4, s["q"], s["k"], s["v"], s["g"], s["beta"], s["parents"], o_off)
            assert ei.value.code == L.ONELA_ERR_ARG
        big = P.custom_steps(15, 1, 2, 64, 64, (5,))[2]
        b = P.to_dev(big)[0]
        with pytest.raises(L.OnelaError) as ei:        # W_max = 4
            dec.step(b["q"], b["k"], b["v"], b["g"], b["beta"], b["parents"])
        assert ei.value.code == L.ONELA_ERR_CAPACITY
        assert dec.status() == 0
    finally:
        dec.close()


@pytest.mark.parametrize("s0_dtype", ["f32", "bf16"])
@pytest.mark.parametrize("W,T,R,H", [(256, 7, 1, 4), (129, 4, 2, 3), (32, 1, 1, 2)])
def test_tc_d256(s0_dtype, W, T, R, H):
    """d_k = d_v = 256 on the tensor cores (two CTAs per beam tile, one per
    half of the rows of S), whole decodes against the fp64 oracle."""
    import linear_attention_beam_shared_b200 as L
    wl, S0, steps = P.custom_steps(60 + W + T, R, H, 256, 256, (W,) * T, parents="mixed" if R > 1 else "zipf")
    S0c = synth.cast_state(S0, s0_dtype)
    gpu, kind = P.run_gpu(S0c, steps, "bf16", L.ONELA_KERNEL_TC)
    assert kind == L.ONELA_KERNEL_TC
    P.compare(gpu, P.oracle(S0c, steps), steps, s0_dtype)


@pytest.mark.parametrize("W,T,R,H", [(129, 4, 2, 3), (256, 6, 1, 2)])
def test_tc_d256_three_terms(W, T, R, H):
    """A three-term split of an fp32 S0 at d = 256: the image (192 KB per CTA)
    streams through the kernel's ring of shared-memory slots, so AUTO keeps
    the tensor-core kernel; whole decodes against the fp64 oracle."""
    import linear_attention_beam_shared_b200 as L
    h = L.onela_create(1, 2, 256, 256, 32, 3, "f32", "bf16", L.ONELA_KERNEL_AUTO, s0_split=3)
    assert L.onela_kernel_kind(h) == L.ONELA_KERNEL_TC
    L.onela_destroy(h)
    wl, S0, steps = P.custom_steps(70 + W + T, R, H, 256, 256, (W,) * T, parents="mixed" if R > 1 else "zipf")
    S0c = synth.cast_state(S0, "f32")
    gpu, kind = P.run_gpu(S0c, steps, "bf16", L.ONELA_KERNEL_TC, s0_split=3)
    assert kind == L.ONELA_KERNEL_TC
    P.compare(gpu, P.oracle(S0c, steps), steps, "f32")
