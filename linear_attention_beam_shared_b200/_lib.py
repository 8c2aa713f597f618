"""Thin ctypes binding of the C ABI in include/onela.h.

Argument marshalling only: every function here checks the tensors it is
given (device, dtype, shape, contiguity), turns them into raw pointers and
calls the function of the same name in ``libonela_b200.so``.  All arithmetic
runs in the library's CUDA kernels.  If the library has not been built the
import fails loudly; there is no fallback.
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional

import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libonela_b200.so")

ONELA_F32, ONELA_BF16 = 0, 1
ONELA_OK, ONELA_ERR_ARG, ONELA_ERR_STATE, ONELA_ERR_CAPACITY = 0, 1, 2, 3
ONELA_ERR_PARENT, ONELA_ERR_CUDA, ONELA_ERR_UNSUPPORTED, ONELA_ERR_SCRATCH = 4, 5, 6, 7
ONELA_ERR_TIMEOUT = 8
ONELA_KERNEL_AUTO, ONELA_KERNEL_SIMT, ONELA_KERNEL_TC = 0, 1, 2
ONELA_FLAG_PDL = 1
ONELA_FLAG_NVTX = 4

_DT = {ONELA_F32: torch.float32, ONELA_BF16: torch.bfloat16}
_DT_CODE = {"f32": ONELA_F32, "bf16": ONELA_BF16, torch.float32: ONELA_F32, torch.bfloat16: ONELA_BF16}


class onela_config(ctypes.Structure):
    _fields_ = [(n, ctypes.c_int32) for n in (
        "R", "H", "d_k", "d_v", "W_max", "T_max", "s0_dtype", "qkv_dtype",
        "kernel", "s0_split", "device", "flags")]


class OnelaError(RuntimeError):
    def __init__(self, code: int, where: str):
        self.code = code
        super().__init__(f"{where}: {error_string(code)} (code {code})")


def _load() -> ctypes.CDLL:
    if not os.path.exists(LIB_PATH):
        raise ImportError(
            f"{LIB_PATH} is missing: build it with "
            "`python linear_attention_beam_shared_b200/build.py` (needs nvcc)")
    lib = ctypes.CDLL(LIB_PATH)
    vp, i32 = ctypes.c_void_p, ctypes.c_int32
    sig = {
        "onela_create": ([ctypes.POINTER(onela_config), ctypes.POINTER(vp)], ctypes.c_int),
        "onela_set_prompt_state": ([vp, vp, vp], ctypes.c_int),
        "onela_prefill": ([vp, i32, vp, vp, vp, vp, vp], ctypes.c_int),
        "onela_read_prompt_state": ([vp, vp, vp], ctypes.c_int),
        "onela_select_scratch_bytes": ([i32, i32, i32, i32], ctypes.c_size_t),
        "onela_select_beams": ([i32, i32, i32, i32, vp, vp, vp, vp, vp, vp, ctypes.c_size_t, i32, vp],
                               ctypes.c_int),
        "onela_decode_step": ([vp, i32, i32, vp, vp, vp, vp, vp, vp, vp, vp], ctypes.c_int),
        "onela_decode_steps": ([vp, i32, vp, vp, vp, vp, vp, vp, vp, vp, vp], ctypes.c_int),
        "onela_set_wait_policy": ([vp, ctypes.c_uint64, i32], ctypes.c_int),
        "onela_set_prefill_segments": ([vp, i32], ctypes.c_int),
        "onela_reset": ([vp, vp], ctypes.c_int),
        "onela_fold": ([vp, i32, vp], ctypes.c_int),
        "onela_read_root_state": ([vp, vp, vp], ctypes.c_int),
        "onela_read_fold_depth": ([vp, vp, vp], ctypes.c_int),
        "onela_status": ([vp, ctypes.POINTER(i32)], ctypes.c_int),
        "onela_destroy": ([vp], ctypes.c_int),
        "onela_read_records": ([vp, i32, vp, vp, vp, vp], ctypes.c_int),
        "onela_read_ancestry": ([vp, i32, vp, vp], ctypes.c_int),
        "onela_steps_done": ([vp], ctypes.c_int),
        "onela_kernel_kind": ([vp], ctypes.c_int),
        "onela_last_call_launches": ([vp], ctypes.c_int),
        "onela_error_string": ([ctypes.c_int], ctypes.c_char_p),
        "onela_decode_step_noalloc": ([ctypes.POINTER(onela_config), i32, i32, i32, vp, vp, vp, vp, vp,
                                       vp, vp, vp, vp, vp], ctypes.c_int),
    }
    for name, (args, res) in sig.items():
        fn = getattr(lib, name)
        fn.argtypes = args
        fn.restype = res
    return lib


lib = _load()


def error_string(code: int) -> str:
    return lib.onela_error_string(int(code)).decode()


def _check(code: int, where: str) -> None:
    if code != ONELA_OK:
        raise OnelaError(code, where)


def _stream(stream) -> ctypes.c_void_p:
    if stream is None:
        stream = torch.cuda.current_stream()
    if isinstance(stream, torch.cuda.Stream):
        return ctypes.c_void_p(stream.cuda_stream)
    return ctypes.c_void_p(int(stream))


def _ptr(t: Optional[torch.Tensor], name: str, dtype=None, shape=None, device=None):
    if t is None:
        return None
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name} must be a torch.Tensor")
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if device is not None and t.device.index != device:
        raise ValueError(f"{name} is on cuda:{t.device.index}, handle is on cuda:{device}")
    if dtype is not None and t.dtype != dtype:
        raise ValueError(f"{name} must be {dtype}, got {t.dtype}")
    if shape is not None and tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name} must have shape {tuple(shape)}, got {tuple(t.shape)}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    return ctypes.c_void_p(t.data_ptr())


class Handle:
    """An ``onela_handle*`` plus the configuration it was made with."""

    def __init__(self, ptr: int, cfg: onela_config):
        self.ptr = ctypes.c_void_p(ptr)
        self.cfg = cfg

    def __repr__(self):
        c = self.cfg
        return (f"Handle(R={c.R}, H={c.H}, d_k={c.d_k}, d_v={c.d_v}, W_max={c.W_max}, "
                f"T_max={c.T_max}, kernel={onela_kernel_kind(self)})")


def onela_create(R: int, H: int, d_k: int, d_v: int, W_max: int, T_max: int,
                 s0_dtype="f32", qkv_dtype="bf16", kernel: int = ONELA_KERNEL_AUTO,
                 s0_split: int = 0, device: int = 0, flags: int = 0) -> Handle:
    cfg = onela_config(R, H, d_k, d_v, W_max, T_max, _DT_CODE[s0_dtype], _DT_CODE[qkv_dtype],
                       kernel, s0_split, device, flags)
    out = ctypes.c_void_p()
    _check(lib.onela_create(ctypes.byref(cfg), ctypes.byref(out)), "onela_create")
    return Handle(out.value, cfg)


def onela_set_prompt_state(h: Handle, S0: torch.Tensor, stream=None) -> None:
    c = h.cfg
    p = _ptr(S0, "S0", _DT[c.s0_dtype], (c.R, c.H, c.d_v, c.d_k), c.device)
    _check(lib.onela_set_prompt_state(h.ptr, p, _stream(stream)), "onela_set_prompt_state")


def onela_prefill(h: Handle, k, v, g, beta, stream=None) -> None:
    """k, v: [R][L][H][d] in the handle's qkv dtype; g, beta: [R][L][H] fp32."""
    c = h.cfg
    dt = _DT[c.qkv_dtype]
    if not isinstance(k, torch.Tensor) or k.dim() != 4:
        raise ValueError("k must be a 4-D tensor [R][L][H][d_k]")
    L = int(k.shape[1])
    args = (
        _ptr(k, "k", dt, (c.R, L, c.H, c.d_k), c.device),
        _ptr(v, "v", dt, (c.R, L, c.H, c.d_v), c.device),
        _ptr(g, "g", torch.float32, (c.R, L, c.H), c.device),
        _ptr(beta, "beta", torch.float32, (c.R, L, c.H), c.device),
    )
    _check(lib.onela_prefill(h.ptr, L, *args, _stream(stream)), "onela_prefill")


def onela_select_beams(beam_score: torch.Tensor, logp: torch.Tensor, W: int, stream=None, out=None):
    """beam_score fp32 [R][W_prev], logp fp32 [R][W_prev][C] on one CUDA device.
    Returns (parent_idx int32 [R][W], token int32 [R][W], score fp32 [R][W]).
    ``out`` = (parent_idx, token, score, scratch) reuses caller tensors (no
    allocation, e.g. inside a captured CUDA graph); scratch is a uint8 tensor
    of at least onela_select_scratch_bytes bytes."""
    if not isinstance(logp, torch.Tensor) or logp.dim() != 3:
        raise ValueError("logp must be a 3-D tensor [R][W_prev][C]")
    R, W_prev, C = (int(x) for x in logp.shape)
    dev = logp.device
    args = (_ptr(beam_score, "beam_score", torch.float32, (R, W_prev), dev.index),
            _ptr(logp, "logp", torch.float32, (R, W_prev, C), dev.index))
    nbytes = int(lib.onela_select_scratch_bytes(R, W_prev, C, int(W)))
    if out is None:
        parent = torch.empty((R, W), dtype=torch.int32, device=dev)
        token = torch.empty((R, W), dtype=torch.int32, device=dev)
        score = torch.empty((R, W), dtype=torch.float32, device=dev)
        scratch = torch.empty(max(nbytes, 16), dtype=torch.uint8, device=dev)
    else:
        parent, token, score, scratch = out
        nbytes = scratch.numel()
    _check(lib.onela_select_beams(R, W_prev, C, int(W), *args, _ptr(parent, "parent"), _ptr(token, "token"),
                                  _ptr(score, "score"), _ptr(scratch, "scratch"), nbytes, dev.index,
                                  _stream(stream)), "onela_select_beams")
    return parent, token, score


def onela_read_prompt_state(h: Handle, stream=None) -> torch.Tensor:
    c = h.cfg
    S0 = torch.empty((c.R, c.H, c.d_v, c.d_k), dtype=_DT[c.s0_dtype], device=torch.device("cuda", c.device))
    _check(lib.onela_read_prompt_state(h.ptr, _ptr(S0, "S0"), _stream(stream)), "onela_read_prompt_state")
    return S0


def onela_decode_step(h: Handle, W_prev: int, W: int, q, k, v, g, beta, parent_idx, o,
                      stream=None) -> None:
    c = h.cfg
    dt = _DT[c.qkv_dtype]
    args = (
        _ptr(q, "q", dt, (c.R, W, c.H, c.d_k), c.device),
        _ptr(k, "k", dt, (c.R, W, c.H, c.d_k), c.device),
        _ptr(v, "v", dt, (c.R, W, c.H, c.d_v), c.device),
        _ptr(g, "g", torch.float32, (c.R, W, c.H), c.device),
        _ptr(beta, "beta", torch.float32, (c.R, W, c.H), c.device),
        _ptr(parent_idx, "parent_idx", torch.int32, (c.R, W), c.device),
        _ptr(o, "o", torch.float32, (c.R, W, c.H, c.d_v), c.device),
    )
    _check(lib.onela_decode_step(h.ptr, int(W_prev), int(W), *args, _stream(stream)),
           "onela_decode_step")


def onela_decode_steps(h: Handle, steps, outs, stream=None) -> None:
    """Several consecutive steps in one call.  steps: list of dicts with the
    step tensors q, k, v, g, beta, parents (the layouts of onela_decode_step);
    outs: list of o tensors (each step's W is its parents' length)."""
    c = h.cfg
    dt = _DT[c.qkv_dtype]
    n = len(steps)
    if n < 1 or len(outs) != n:
        raise ValueError("steps and outs must be non-empty lists of the same length")
    Ws = [int(s["parents"].shape[-1]) for s in steps]
    arrs = {name: (ctypes.c_void_p * n)() for name in ("q", "k", "v", "g", "beta", "parents", "o")}
    for i, (s, o, W) in enumerate(zip(steps, outs, Ws)):
        arrs["q"][i] = _ptr(s["q"], "q", dt, (c.R, W, c.H, c.d_k), c.device).value
        arrs["k"][i] = _ptr(s["k"], "k", dt, (c.R, W, c.H, c.d_k), c.device).value
        arrs["v"][i] = _ptr(s["v"], "v", dt, (c.R, W, c.H, c.d_v), c.device).value
        arrs["g"][i] = _ptr(s["g"], "g", torch.float32, (c.R, W, c.H), c.device).value
        arrs["beta"][i] = _ptr(s["beta"], "beta", torch.float32, (c.R, W, c.H), c.device).value
        arrs["parents"][i] = _ptr(s["parents"], "parent_idx", torch.int32, (c.R, W), c.device).value
        arrs["o"][i] = _ptr(o, "o", torch.float32, (c.R, W, c.H, c.d_v), c.device).value
    Wa = (ctypes.c_int32 * n)(*Ws)
    _check(lib.onela_decode_steps(h.ptr, n, Wa, arrs["q"], arrs["k"], arrs["v"], arrs["g"], arrs["beta"],
                                  arrs["parents"], arrs["o"], _stream(stream)), "onela_decode_steps")


def onela_set_wait_policy(h: Handle, limit_ns: int, stall: bool = False) -> None:
    _check(lib.onela_set_wait_policy(h.ptr, int(limit_ns), 1 if stall else 0), "onela_set_wait_policy")


def onela_set_prefill_segments(h: Handle, segments: int) -> None:
    _check(lib.onela_set_prefill_segments(h.ptr, int(segments)), "onela_set_prefill_segments")


def onela_reset(h: Handle, stream=None) -> None:
    _check(lib.onela_reset(h.ptr, _stream(stream)), "onela_reset")


def onela_fold(h: Handle, max_depth: int, stream=None) -> None:
    _check(lib.onela_fold(h.ptr, int(max_depth), _stream(stream)), "onela_fold")


def onela_read_root_state(h: Handle, stream=None) -> torch.Tensor:
    c = h.cfg
    S = torch.empty((c.R, c.H, c.d_v, c.d_k), dtype=_DT[c.s0_dtype], device=torch.device("cuda", c.device))
    _check(lib.onela_read_root_state(h.ptr, _ptr(S, "S"), _stream(stream)), "onela_read_root_state")
    return S


def onela_read_fold_depth(h: Handle, stream=None) -> torch.Tensor:
    c = h.cfg
    d = torch.empty((c.R,), dtype=torch.int32, device=torch.device("cuda", c.device))
    _check(lib.onela_read_fold_depth(h.ptr, _ptr(d, "depth"), _stream(stream)), "onela_read_fold_depth")
    return d


def onela_status(h: Handle) -> int:
    """Synchronises the device; returns the error word, raises on an error."""
    word = ctypes.c_int32(0)
    _check(lib.onela_status(h.ptr, ctypes.byref(word)), "onela_status")
    return word.value


def onela_status_code(h: Handle):
    """(return code, error word) without raising."""
    word = ctypes.c_int32(0)
    rc = lib.onela_status(h.ptr, ctypes.byref(word))
    return rc, word.value


def onela_destroy(h: Handle) -> None:
    if h.ptr:
        _check(lib.onela_destroy(h.ptr), "onela_destroy")
        h.ptr = ctypes.c_void_p()


def onela_read_records(h: Handle, t: int, W_t: int, stream=None):
    """Records of depth t as new tensors: alpha [R][H][W_t], delta
    [R][H][W_t][d_v], k [R][H][W_t][d_k]."""
    c = h.cfg
    dev = torch.device("cuda", c.device)
    alpha = torch.empty((c.R, c.H, W_t), dtype=torch.float32, device=dev)
    delta = torch.empty((c.R, c.H, W_t, c.d_v), dtype=torch.float32, device=dev)
    k = torch.empty((c.R, c.H, W_t, c.d_k), dtype=_DT[c.qkv_dtype], device=dev)
    _check(lib.onela_read_records(h.ptr, int(t), _ptr(alpha, "alpha"), _ptr(delta, "delta"),
                                  _ptr(k, "k"), _stream(stream)), "onela_read_records")
    return alpha, delta, k


def onela_read_ancestry(h: Handle, t: int, W_t: int, stream=None) -> torch.Tensor:
    c = h.cfg
    anc = torch.zeros((c.R, W_t, max(t - 1, 0)), dtype=torch.int32,
                      device=torch.device("cuda", c.device))
    if t > 1:
        _check(lib.onela_read_ancestry(h.ptr, int(t), _ptr(anc, "anc"), _stream(stream)),
               "onela_read_ancestry")
    return anc


def onela_steps_done(h: Handle) -> int:
    return int(lib.onela_steps_done(h.ptr))


def onela_kernel_kind(h: Handle) -> int:
    return int(lib.onela_kernel_kind(h.ptr))


def onela_last_call_launches(h: Handle) -> int:
    return int(lib.onela_last_call_launches(h.ptr))


def onela_decode_step_noalloc(R: int, H: int, d_k: int, d_v: int, W_max: int, T_max: int,
                              s0_dtype, qkv_dtype, t: int, W_prev: int, W: int, S0, q, k, v, g,
                              beta, parent_idx, o, status, device: int = 0, stream=None) -> None:
    """Decode step t that allocates no device memory (state in the library's
    fixed 32 MiB array).  status: int32 CUDA tensor of one element, written
    with the error word."""
    cfg = onela_config(R, H, d_k, d_v, W_max, T_max, _DT_CODE[s0_dtype], _DT_CODE[qkv_dtype],
                       0, 0, device)
    dt = _DT[cfg.qkv_dtype]
    args = (
        _ptr(S0, "S0", _DT[cfg.s0_dtype], (R, H, d_v, d_k), device),
        _ptr(q, "q", dt, (R, W, H, d_k), device),
        _ptr(k, "k", dt, (R, W, H, d_k), device),
        _ptr(v, "v", dt, (R, W, H, d_v), device),
        _ptr(g, "g", torch.float32, (R, W, H), device),
        _ptr(beta, "beta", torch.float32, (R, W, H), device),
        _ptr(parent_idx, "parent_idx", torch.int32, (R, W), device),
        _ptr(o, "o", torch.float32, (R, W, H, d_v), device),
        _ptr(status, "status", torch.int32, (1,), device),
    )
    _check(lib.onela_decode_step_noalloc(ctypes.byref(cfg), int(t), int(W_prev), int(W), *args,
                                         _stream(stream)), "onela_decode_step_noalloc")
