"""Shared-state Gated DeltaNet beam decode for B200 (sm_100a).

One GDN decode step for W beams that share one prompt-derived state S0 per
(request, head): beams are chains of append-only transition records
(alpha, delta, k) reached through an ancestry index, and S_{t-1}[k; q] is
formed as S0 [k; q] (S0 read once, shared by all beams) plus a gated replay
over the beam's ancestor records (OneLA abstract; evolve.pub review, key
claims on section 3.2, equations 2-4).

The work runs in the CUDA library ``libonela_b200.so`` (C ABI in
``include/onela.h``); this package is its Python binding.  ``onela_*``
functions mirror the C entry points one to one; ``BeamDecoder`` is a small
convenience wrapper around a handle.
"""
from __future__ import annotations

import torch

from . import _lib
from ._lib import (  # noqa: F401
    ONELA_BF16, ONELA_ERR_ARG, ONELA_ERR_CAPACITY, ONELA_ERR_CUDA, ONELA_ERR_PARENT,
    ONELA_ERR_STATE, ONELA_ERR_UNSUPPORTED, ONELA_F32, ONELA_FLAG_NVTX, ONELA_FLAG_PDL, ONELA_KERNEL_AUTO, ONELA_KERNEL_SIMT,
    ONELA_ERR_SCRATCH, ONELA_ERR_TIMEOUT, ONELA_KERNEL_TC, ONELA_OK, Handle, OnelaError, error_string, onela_create,
    onela_decode_step, onela_decode_step_noalloc, onela_decode_steps, onela_set_wait_policy, onela_set_prefill_segments, onela_destroy, onela_fold, onela_kernel_kind, onela_last_call_launches, onela_prefill,
    onela_read_ancestry, onela_read_fold_depth, onela_read_prompt_state, onela_read_records,
    onela_read_root_state, onela_reset, onela_select_beams, onela_set_prompt_state,
    onela_status, onela_status_code, onela_steps_done,
)

LIB_PATH = _lib.LIB_PATH


class BeamDecoder:
    """Owns one handle; tracks the beam count of the previous step."""

    def __init__(self, R, H, d_k, d_v, W_max, T_max, s0_dtype="f32", qkv_dtype="bf16",
                 kernel=ONELA_KERNEL_AUTO, s0_split=0, device=0, flags=0):
        self.h = onela_create(R, H, d_k, d_v, W_max, T_max, s0_dtype, qkv_dtype, kernel,
                              s0_split, device, flags)
        self.device = torch.device("cuda", device)
        self.W_prev = 1
        self.Ws = []

    @property
    def kernel(self) -> int:
        return onela_kernel_kind(self.h)

    def set_prompt_state(self, S0, stream=None):
        onela_set_prompt_state(self.h, S0, stream)
        self.W_prev, self.Ws = 1, []

    def prefill(self, k, v, g, beta, stream=None):
        """Build S0 on the device from a prompt (see onela_prefill)."""
        onela_prefill(self.h, k, v, g, beta, stream)
        self.W_prev, self.Ws = 1, []

    def prompt_state(self, stream=None):
        return onela_read_prompt_state(self.h, stream)

    def step(self, q, k, v, g, beta, parent_idx, o=None, stream=None):
        c = self.h.cfg
        W = int(parent_idx.shape[-1])
        if o is None:
            o = torch.empty((c.R, W, c.H, c.d_v), dtype=torch.float32, device=self.device)
        onela_decode_step(self.h, self.W_prev, W, q, k, v, g, beta, parent_idx, o, stream)
        self.W_prev = W
        self.Ws.append(W)
        return o

    def steps(self, steps, outs=None, stream=None):
        """Several consecutive steps in one call (see onela_decode_steps):
        steps is a list of dicts with q, k, v, g, beta, parents."""
        c = self.h.cfg
        if outs is None:
            outs = [torch.empty((c.R, int(s["parents"].shape[-1]), c.H, c.d_v), dtype=torch.float32,
                                device=self.device) for s in steps]
        onela_decode_steps(self.h, steps, outs, stream)
        for s in steps:
            W = int(s["parents"].shape[-1])
            self.W_prev = W
            self.Ws.append(W)
        return outs

    def prefill_segments(self, segments: int) -> None:
        """Segments of the chunked tensor-core prefill (0: automatic)."""
        onela_set_prefill_segments(self.h, segments)

    def last_launches(self) -> int:
        """Kernel launches of the last decode or prefill call."""
        return onela_last_call_launches(self.h)

    def reset(self, stream=None):
        onela_reset(self.h, stream)
        self.W_prev, self.Ws = 1, []

    def fold(self, max_depth=None, stream=None):
        """Fold each request's shared ancestor prefix (down to max_depth,
        default: as deep as it goes) into its root state (see onela_fold)."""
        onela_fold(self.h, len(self.Ws) if max_depth is None else max_depth, stream)

    def root_state(self, stream=None):
        return onela_read_root_state(self.h, stream)

    def fold_depth(self, stream=None):
        return onela_read_fold_depth(self.h, stream)

    def status(self) -> int:
        return onela_status(self.h)

    def records(self, t: int):
        return onela_read_records(self.h, t, self.Ws[t - 1])

    def ancestry(self, t: int):
        return onela_read_ancestry(self.h, t, self.Ws[t - 1])

    def close(self):
        onela_destroy(self.h)

    def __del__(self):  # pragma: no cover - best effort
        try:
            if self.h.ptr:
                onela_destroy(self.h)
        except Exception:
            pass
