"""onela_decode_step_noalloc: the decode step for callers that cannot
allocate device memory (inside a stream capture, or inside an engine that
owns all device memory and hands its plug-ins only their tensors).  It keeps
its state in the library's fixed 32 MiB device array, so these tests check
that it gives what the handle-based onela_decode_step gives, decode after
decode, with nothing left over from an earlier call spoiling a later one.

This file is collected last on purpose: it is the newest entry point, and a
run that stops at its first failure has then already run every other test.
"""
import ctypes

import numpy as np
import pytest
import torch

import synth
from tests import _parity as P


def _noalloc_decode(L, S0, dsteps, R, H, d, W_max, T_max, s0_dtype, qkv, status):
    outs = []
    W_prev = 1
    for t, s in enumerate(dsteps, start=1):
        o = torch.full((R, s["W"], H, d), float("nan"), device="cuda")
        L.onela_decode_step_noalloc(R, H, d, d, W_max, T_max, s0_dtype, qkv, t, W_prev, s["W"], S0,
                                    s["q"], s["k"], s["v"], s["g"], s["beta"], s["parents"], o, status)
        outs.append(o)
        W_prev = s["W"]
    torch.cuda.synchronize()
    return [o.cpu() for o in outs]


@pytest.mark.gpu
@pytest.mark.parametrize("s0_dtype,qkv,d,Ws,R,H", [
    ("f32", "bf16", 128, (16, 96, 96, 64), 1, 4),
    ("bf16", "bf16", 64, (8, 40, 33), 2, 3),
    ("f32", "f32", 64, (8, 8, 8), 1, 2),
])
def test_noalloc_matches_handle_path(s0_dtype, qkv, d, Ws, R, H):
    import linear_attention_beam_shared_b200 as L
    wl, S0, steps = P.custom_steps(41 + d, R, H, d, d, Ws, qkv_dtype=qkv,
                                   parents="mixed" if R > 1 else "zipf")
    S0c = synth.cast_state(S0, s0_dtype)
    ref, _ = P.run_gpu(S0c, steps, qkv, L.ONELA_KERNEL_SIMT, read_back=False)
    fp64 = P.oracle(S0c, steps)
    dsteps = P.to_dev(steps)
    status = torch.full((1,), -1, dtype=torch.int32, device="cuda")
    tol = P.TOL[s0_dtype]
    # Two decodes in a row through the same array: the second must not see
    # anything the first left behind.  The same SIMT kernel on the same
    # inputs as the handle path, so the outputs agree bit for bit; every
    # step's o (which depends on the delta records of all its ancestors) is
    # also held to the fp64 oracle at the decode tolerance.
    for _ in range(2):
        outs = _noalloc_decode(L, S0c.cuda(), dsteps, R, H, d, max(Ws), len(Ws), s0_dtype, qkv, status)
        assert int(status.item()) == 0
        for a, b, f in zip(outs, ref, fp64):
            assert torch.equal(a, b["o"])
            assert float(np.abs(a.double().numpy() - f["o"]).max()) <= tol


@pytest.mark.gpu
def test_noalloc_two_calls_in_a_row_and_parent_error():
    """Two consecutive steps; a bad parent in the second sets bit 0 of the
    status, and the next decode (t = 1) starts clean again."""
    import linear_attention_beam_shared_b200 as L
    wl, S0, steps = P.custom_steps(43, 1, 2, 64, 64, (6, 6))
    S0c = synth.cast_state(S0, "f32").cuda()
    ref, _ = P.run_gpu(S0c.cpu(), steps, "bf16", L.ONELA_KERNEL_SIMT, read_back=False)
    d = P.to_dev(steps)
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    outs = _noalloc_decode(L, S0c, d, 1, 2, 64, 6, 2, "f32", "bf16", status)
    assert int(status.item()) == 0
    for a, b in zip(outs, ref):
        assert torch.equal(a, b["o"])
    bad = dict(d[1])
    bad["parents"] = d[1]["parents"].clone()
    bad["parents"][0, 2] = 6
    _noalloc_decode(L, S0c, [d[0], bad], 1, 2, 64, 6, 2, "f32", "bf16", status)
    assert int(status.item()) & 1
    outs = _noalloc_decode(L, S0c, d, 1, 2, 64, 6, 2, "f32", "bf16", status)
    assert int(status.item()) == 0
    fp64 = P.oracle(S0c.cpu(), steps)
    for a, b, f in zip(outs, ref, fp64):
        assert torch.equal(a, b["o"])
        assert float(np.abs(a.double().numpy() - f["o"]).max()) <= P.TOL["f32"]


def test_noalloc_rejects_oversize_and_bad_steps_on_the_host():
    """Checked before any CUDA call, so this runs without a GPU."""
    import linear_attention_beam_shared_b200 as L
    lib = L._lib.lib
    dummy = ctypes.c_void_p(16)   # never dereferenced: the calls fail validation first
    args = [dummy] * 10

    def call(cfg, t, W_prev, W):
        return lib.onela_decode_step_noalloc(ctypes.byref(cfg), t, W_prev, W, *args)

    big = L._lib.onela_config(4, 32, 128, 128, 512, 8, 0, 1, 0, 0, 0)
    assert call(big, 1, 1, 512) == L.ONELA_ERR_SCRATCH
    small = L._lib.onela_config(1, 2, 64, 64, 8, 3, 0, 1, 0, 0, 0)
    assert call(small, 0, 1, 8) == L.ONELA_ERR_ARG      # t starts at 1
    assert call(small, 4, 8, 8) == L.ONELA_ERR_ARG      # beyond T_max
    assert call(small, 1, 2, 8) == L.ONELA_ERR_ARG      # W_prev must be 1 at t = 1
    assert call(small, 2, 8, 9) == L.ONELA_ERR_ARG      # beyond W_max
    assert lib.onela_decode_step_noalloc(None, 1, 1, 1, *args) == L.ONELA_ERR_ARG
