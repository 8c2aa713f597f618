#!/usr/bin/env python
"""Benchmark: shared-state GDN beam decode on B200.

One benchmark step = one whole T-step beam decode of the workload (every
decode step of the hot path: ancestry update, S0 [K; Q] products, replay,
epilogue, record append), captured once in a CUDA graph and replayed.  L2 is
flushed (a 512 MiB write) before every timed step, outside the timed events.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
                    [--workload long5k] [--kernel auto|simt|tc]

Multi-GPU (launched by torchrun): every rank decodes its own request (its own
S0 and inputs) with no collective on the data path; value = all ranks' beam.head
steps / max-over-ranks device time ("weak" scaling).

``--impl reference`` times the fp64 CPU oracle (the plain-C full-state beam
tree) on the host cores for the same workload, metric and unit.
"""
from __future__ import annotations

import argparse
import hashlib

import json
import os
import statistics
import subprocess
import sys
import tempfile
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import synth  # noqa: E402

METRIC = "GDN beam·head decode steps/s at W=256,T=7; % of HBM/tensor roofline"
UNIT = "beam·head steps/s"


# ------------------------------------------------------------------ helpers
def dist_env():
    ws = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return ws, rank, local


def rank_workload(base, rank):
    """Every rank decodes its own request: the same shapes, its own S0 and
    inputs (its own random stream)."""
    return base.replace(seed_id=base.seed_id + 1000 * rank)


def max_over_ranks(x, device):
    """The largest value of x over all ranks (x itself with one rank).  The
    tensor lives on ``device``: the GPU for NCCL, the CPU for gloo."""
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return float(x)
    t = torch.tensor([float(x)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def whole_job_value(units_per_rank, ws, max_ms_per_step):
    """Whole-job throughput: the units all ranks processed / the slowest
    rank's device time."""
    return units_per_rank * ws / (max_ms_per_step / 1e3)


def measured_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            d = json.load(f)
        return float(d["hbm_gbs"]), float(d["bf16_tflops"]), float(d.get("bf16_tflops_sustained", 0)), "measured"
    return 6650.0, 1590.0, 1400.0, "fallback"


KERNEL_SOURCES = {"tc": "step_tc.cu", "simt": "step_simt.cu"}


def kernel_source_hash(kind="tc"):
    """Hash of the decode kernel's source file (step_tc.cu or step_simt.cu)
    with comments and blank lines removed, so that a change of wording, or a
    change to another kernel of the library, keeps the recorded counters
    valid."""
    import re
    h = hashlib.sha256()
    for p in [os.path.join(ROOT, "linear_attention_beam_shared_b200", "csrc", KERNEL_SOURCES[kind])]:
        with open(p, "r", encoding="utf-8", errors="replace") as f:
            text = f.read()
        text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
        text = "\n".join(line.split("//")[0].rstrip() for line in text.splitlines() if line.split("//")[0].strip())
        h.update(os.path.basename(p).encode())
        h.update(text.encode())
    return h.hexdigest()[:16]


def ncu_traffic(kernel_kind):
    """DRAM bytes per launch of the decode kernel from the committed ncu
    summary, or None when the kernel sources changed since it was taken."""
    path = os.path.join(ROOT, "profiles", "ncu_traffic.json")
    if not os.path.exists(path):
        return None
    with open(path) as f:
        d = json.load(f)
    entry = d.get(kernel_kind)
    if not entry or entry.get("source_hash") != kernel_source_hash(kernel_kind):
        return None
    return entry


def s0_by_prefill_gpu(wl, device):
    """S0 for the workload: the GDN recurrence from zero over its synthetic
    prompt, run with plain torch fp64 ops on the device (input synthesis for
    the benchmark only; not part of the timed decode)."""
    k, v, a, b = synth.draw_prompt(wl)
    k = torch.from_numpy(k).to(device)
    v = torch.from_numpy(v).to(device)
    a = torch.from_numpy(a).to(device)
    b = torch.from_numpy(b).to(device)
    R, L, H, dk = k.shape
    S = torch.zeros((R, H, wl.d_v, dk), dtype=torch.float64, device=device)
    for l in range(L):
        kl, vl = k[:, l], v[:, l]
        al, bl = a[:, l, :, None], b[:, l, :, None]
        u = torch.einsum("rhij,rhj->rhi", S, kl)
        delta = bl * (vl - al * u)
        S = al[..., None] * S + delta[..., :, None] * kl[..., None, :]
    S32 = S.float().cpu()
    return S32.to(torch.bfloat16) if wl.s0_dtype == "bf16" else S32


# FP32 lanes per SM and SM count of the B200, for the ALU roofline of the
# prefill (its recurrence runs on the CUDA cores in fp32).
FP32_LANES_PER_SM, N_SMS = 128, 148


def time_prefill(wl, device, stream, flush, reps=10, warmup=3):
    """Device time of onela_prefill over the workload's prompt (every request
    and head), L2 flushed before each call; and the oracle's prefill on a
    bounded host sample.  Returns the JSON object for the bench line."""
    import linear_attention_beam_shared_b200 as L
    from oracle import gdn
    k, v, a, b = synth.draw_prompt(wl)
    kd = synth.cast_vec(k, wl.qkv_dtype).to(device)
    vd = synth.cast_vec(v, wl.qkv_dtype).to(device)
    g = torch.from_numpy(np.log(a)).float().to(device)
    beta = torch.from_numpy(b).float().to(device)
    dec = L.BeamDecoder(wl.R, wl.H, wl.d_k, wl.d_v, wl.W, wl.T, wl.s0_dtype, wl.qkv_dtype, device=device.index)
    with torch.cuda.stream(stream):
        dec.prefill(kd, vd, g, beta, stream=stream)
    stream.synchronize()
    launches = dec.last_launches()
    chunked = launches == 4   # prep, segment chains, combine, S0 image
    graph = torch.cuda.CUDAGraph()   # the launches alone, without the host's call overhead
    with torch.cuda.graph(graph, stream=stream):
        dec.prefill(kd, vd, g, beta, stream=stream)
    with torch.cuda.stream(stream):
        for _ in range(warmup):
            flush.fill_(5)
            graph.replay()
    stream.synchronize()
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(reps)]
    with torch.cuda.stream(stream):
        for i, (e0, e1) in enumerate(ev):
            flush.fill_(i & 0xFF)
            e0.record(stream)
            graph.replay()
            e1.record(stream)
    stream.synchronize()
    del graph
    assert dec.status() == 0
    dec.close()
    ms = max_over_ranks(sum(e0.elapsed_time(e1) for e0, e1 in ev) / reps, device)
    units = wl.R * wl.L_prompt * wl.H
    flops = 4.0 * wl.d_k * wl.d_v * units
    peak = N_SMS * FP32_LANES_PER_SM * 2 * 1.965e9 / 1e9   # GFLOP/s at the 1965 MHz boost clock
    achieved = flops / (ms / 1e3) / 1e9
    e = 2 if wl.qkv_dtype == "bf16" else 4
    bytes_ = units * (wl.d_k + wl.d_v) * e + units * 8 + wl.R * wl.H * wl.d_k * wl.d_v * (2 if wl.s0_dtype == "bf16" else 4)
    # The oracle on the host: one head, the first 512 tokens.
    Ls = min(512, wl.L_prompt)
    t0 = time.perf_counter()
    gdn.prefill(k[0, :Ls, :1], v[0, :Ls, :1], a[0, :Ls, :1], b[0, :Ls, :1])
    el = time.perf_counter() - t0
    if chunked:
        # The chunked path's tensor-core work per 64-token chunk and head:
        # Y = S K^T (3 terms), Delta = Z T^T (6 term pairs), dS = Delta~ K
        # (3 terms), twice for the segments after the first (their
        # transition chains), plus the key Gram of the prep kernel.
        C = 64
        nch = (wl.L_prompt + C - 1) // C
        per_chunk = 2 * 128 * (3 * C * wl.d_k + 6 * C * C + 3 * C * wl.d_k)
        # the library's default segmentation: one chain per SM, at least 4 chunks per segment
        nseg = max(1, min((148 // max(1, wl.R * wl.H) + 1) // 2, max(1, nch // 4), nch, 16))
        cps = -(-nch // nseg)
        chunk_chains = nch + (nch - min(cps, nch))   # segments after the first also run their transition chain
        tc_flops = (per_chunk * chunk_chains + 2 * 2 * C * 2 * C * wl.d_k * (-(-nch // 2))) * wl.R * wl.H
        tpeak = measured_peaks()[1] * 1e3                 # GFLOP/s, burst
        roof = {"bound": "tensor", "achieved": round(achieved, 1), "peak": round(tpeak, 1), "unit": "GFLOP/s",
                "frac": round(achieved / tpeak, 4),
                "peak_source": "measured (MEASURED_PEAKS.json bf16_tflops)",
                "note": "achieved = the recurrence's 4 L d^2 H FLOPs / time; the tensor cores execute about "
                        f"{tc_flops / (ms / 1e3) / 1e12:.1f} TFLOP/s with the bf16 term expansion",
                "fp32_alu_frac": round(achieved / peak, 4),
                "hbm_bytes": int(bytes_), "hbm_frac": round(bytes_ / (ms / 1e3) / 1e9 / measured_peaks()[0], 4)}
    else:
        roof = {"bound": "alu", "achieved": round(achieved, 1), "peak": round(peak, 1), "unit": "GFLOP/s",
                "frac": round(achieved / peak, 4),
                "peak_source": "148 SMs x 128 fp32 lanes x 2 FLOP x 1965 MHz",
                "hbm_bytes": int(bytes_), "hbm_frac": round(bytes_ / (ms / 1e3) / 1e9 / measured_peaks()[0], 4)}
    return {
        "workload": f"{wl.name} prompt: R={wl.R}, L={wl.L_prompt}, H={wl.H}, d_k=d_v={wl.d_k}, "
                    f"k/v {wl.qkv_dtype}, S0 {wl.s0_dtype}",
        "path": "chunked on the tensor cores (64-token chunks, segments side by side)" if chunked else "token by token",
        "launches": launches,
        "ms": round(ms, 4), "value": round(units / (ms / 1e3), 1), "unit": "prompt token·head steps/s",
        "roofline": roof,
        "cpu_baseline": {"value": round(Ls / el, 1), "unit": "prompt token·head steps/s", "cores": 1,
                         "kind": "oracle", "sample": f"one head, first {Ls} tokens, numpy fp64 prefill, {el:.2f} s"},
    }


def time_select(device, stream, flush, R=1, W_prev=256, C=256, W=256, reps=20, warmup=3):
    """Device time of onela_select_beams for one decode step's beam set
    (W_prev beams x C children -> W), L2 flushed before each call; the
    oracle's selection on the host for the same inputs.  Returns the JSON
    object for the bench line."""
    import linear_attention_beam_shared_b200 as L
    from oracle import beam
    rng = np.random.default_rng(77)
    bs = (-rng.exponential(3.0, (R, W_prev))).astype(np.float32)
    lp = np.log(rng.dirichlet(np.ones(C), (R, W_prev))).astype(np.float32)
    bsd, lpd = torch.from_numpy(bs).to(device), torch.from_numpy(lp).to(device)
    out = (torch.empty((R, W), dtype=torch.int32, device=device), torch.empty((R, W), dtype=torch.int32, device=device),
           torch.empty((R, W), dtype=torch.float32, device=device),
           torch.empty(int(L._lib.lib.onela_select_scratch_bytes(R, W_prev, C, W)), dtype=torch.uint8, device=device))
    with torch.cuda.stream(stream):
        L.onela_select_beams(bsd, lpd, W, stream=stream, out=out)
    stream.synchronize()
    graph = torch.cuda.CUDAGraph()   # the launches alone, without the host's call overhead
    with torch.cuda.graph(graph, stream=stream):
        L.onela_select_beams(bsd, lpd, W, stream=stream, out=out)
    with torch.cuda.stream(stream):
        for _ in range(warmup):
            flush.fill_(7)
            graph.replay()
    stream.synchronize()
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(reps)]
    with torch.cuda.stream(stream):
        for i, (e0, e1) in enumerate(ev):
            flush.fill_(i & 0xFF)
            e0.record(stream)
            graph.replay()
            e1.record(stream)
    stream.synchronize()
    del graph
    ms = max_over_ranks(sum(e0.elapsed_time(e1) for e0, e1 in ev) / reps, device)
    ref = beam.select_beams(bs, lp, W)
    assert all(np.array_equal(o.cpu().numpy(), r) for o, r in zip(out[:2], ref[:2])), "selection differs from the oracle"
    bytes_ = R * W_prev * C * 4 + R * W_prev * 4 + R * W * 12
    t0 = time.perf_counter()
    reps_cpu = 0
    while time.perf_counter() - t0 < 1.0:
        beam.select_beams(bs, lp, W)
        reps_cpu += 1
    el = time.perf_counter() - t0
    hbm = measured_peaks()[0]
    return {
        "workload": f"R={R}, W_prev={W_prev} beams x C={C} children -> W={W}, fp32 scores",
        "ms": round(ms, 5), "value": round(R * W_prev * C / (ms / 1e3), 1), "unit": "candidates/s",
        "roofline": {"bound": "hbm", "achieved": round(bytes_ / (ms / 1e3) / 1e9, 2), "peak": hbm, "unit": "GB/s",
                     "frac": round(bytes_ / (ms / 1e3) / 1e9 / hbm, 5), "alg_bytes": bytes_},
        "launches": 2,
        "cpu_baseline": {"value": round(R * W_prev * C * reps_cpu / el, 1), "unit": "candidates/s", "cores": 1,
                         "kind": "oracle", "sample": f"the same inputs x{reps_cpu} in {el:.2f} s, numpy sort"},
    }


def time_fold(wl, S0, kernel, device, stream, flush, T=16, every=4, reps=10, warmup=3, alone=True, tmax=None):
    """Folding on a deeper decode: the workload's shapes over T steps, every
    beam of steps every, 2 every, ... a child of one beam (the beam sets
    narrow to one shared ancestor), decoded as one CUDA graph with a fold
    right after each such step and, for comparison, without folds; then the
    fold alone (after the first narrowing step, caches flushed).  The folded
    and unfolded outputs must agree to fp32 rounding.  tmax < T: a record
    store of tmax depths, which only the folded decode can run through.
    Returns the JSON object for the bench line."""
    import linear_attention_beam_shared_b200 as L
    wd = wl.replace(name=wl.name + "_deep", T=T)
    steps = synth.draw_decode(wd)
    narrow = list(range(every - 1, T - 1, every))            # 0-based steps
    for i in narrow:
        steps[i]["parents"] = torch.zeros_like(steps[i]["parents"])
    fold_after = {i + 1 for i in narrow}                     # fold after these steps (1-based)
    dsteps = [{k: (v.to(device) if isinstance(v, torch.Tensor) else v) for k, v in st.items()} for st in steps]

    def make(fold):
        outs = [torch.empty((wd.R, st["W"], wd.H, wd.d_v), dtype=torch.float32, device=device) for st in steps]
        # The folded decode runs through the record store of tmax depths; the
        # unfolded one needs all T of them.
        dec = L.BeamDecoder(wd.R, wd.H, wd.d_k, wd.d_v, wd.W, (tmax or T) if fold else T, wd.s0_dtype, wd.qkv_dtype,
                            kernel=kernel, device=device.index, flags=L.ONELA_FLAG_PDL)
        kernels[fold] = dec.kernel
        dec.set_prompt_state(S0.to(device))

        def run():
            for t, (st, o) in enumerate(zip(dsteps, outs), start=1):
                dec.step(st["q"], st["k"], st["v"], st["g"], st["beta"], st["parents"], o=o, stream=stream)
                if fold and t in fold_after:
                    dec.fold(stream=stream)
        with torch.cuda.stream(stream):
            run()
        stream.synchronize()
        assert dec.status() == 0
        depth = dec.fold_depth(stream).cpu().tolist()
        dec.reset(stream)
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=stream):
            run()
        dec.reset(stream)
        return dec, g, outs, depth

    def timed(graphs, pre=None):
        for _ in range(warmup):
            with torch.cuda.stream(stream):
                if pre is not None:
                    pre.replay()
                flush.fill_(5)
                graphs.replay()
        stream.synchronize()
        ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(reps)]
        with torch.cuda.stream(stream):
            for i, (e0, e1) in enumerate(ev):
                if pre is not None:
                    pre.replay()
                flush.fill_(i & 0xFF)
                e0.record(stream)
                graphs.replay()
                e1.record(stream)
        stream.synchronize()
        return max_over_ranks(sum(e0.elapsed_time(e1) for e0, e1 in ev) / reps, device)

    res, kernels = {}, {}
    for fold in (True, False):
        dec, g, outs, depth = make(fold)
        ms = timed(g)
        res[fold] = (ms, [o.clone() for o in outs], depth)
        del g
        dec.close()
    diff = max(float((a - b).abs().max()) for a, b in zip(res[True][1], res[False][1]))
    scale = max(float(b.abs().max()) for b in res[False][1])
    assert diff <= 2e-5 * max(1.0, scale), f"folded decode differs from the unfolded one by {diff}"
    if tmax and tmax < T:
        names = {L.ONELA_KERNEL_TC: "tc", L.ONELA_KERNEL_SIMT: "simt"}
        return {
            "workload": f"{wl.name} shapes over T={T} steps (R={wd.R}, H={wd.H}, d={wd.d_k}, W={wd.W}), every beam of "
                        f"steps {', '.join(str(i + 1) for i in narrow)} a child of beam 0; folded: folds right after "
                        f"them through a record store of {tmax} depths; unfolded: a store of {T} depths",
            "ms_per_decode": {"folded": round(res[True][0], 5), "unfolded": round(res[False][0], 5)},
            "speedup": round(res[False][0] / res[True][0], 3),
            "record_store_depths": {"folded": tmax, "unfolded": T},
            "kernel": {"folded": names.get(kernels[True]), "unfolded": names.get(kernels[False])},
            "us_per_step": {"folded": round(res[True][0] * 1e3 / T, 3), "unfolded": round(res[False][0] * 1e3 / T, 3)},
            "fold_depth_at_end": res[True][2],
            "max_abs_diff_folded_vs_unfolded": diff,
        }

    out = {
        "workload": f"{wl.name} shapes over T={T} steps (R={wd.R}, H={wd.H}, d={wd.d_k}, W={wd.W}), every beam of "
                    f"steps {', '.join(str(i + 1) for i in narrow)} a child of beam 0; folds right after them",
        "ms_per_decode": {"folded": round(res[True][0], 5), "unfolded": round(res[False][0], 5)},
        "speedup": round(res[False][0] / res[True][0], 3),
        "replayed_depths_max": {"folded": every, "unfolded": T - 1},
        "fold_depth_at_end": res[True][2],
        "max_abs_diff_folded_vs_unfolded": diff,
    }
    if not alone:
        return out
    # The fold alone: steps 1..every (one graph), then the fold (another).
    dec = L.BeamDecoder(wd.R, wd.H, wd.d_k, wd.d_v, wd.W, T, wd.s0_dtype, wd.qkv_dtype, kernel=kernel,
                        device=device.index, flags=L.ONELA_FLAG_PDL)
    dec.set_prompt_state(S0.to(device))
    outs = [torch.empty((wd.R, st["W"], wd.H, wd.d_v), dtype=torch.float32, device=device) for st in steps]
    g_steps, g_fold = torch.cuda.CUDAGraph(), torch.cuda.CUDAGraph()
    with torch.cuda.graph(g_steps, stream=stream):
        for st, o in zip(dsteps[:every], outs):
            dec.step(st["q"], st["k"], st["v"], st["g"], st["beta"], st["parents"], o=o, stream=stream)
    with torch.cuda.graph(g_fold, stream=stream):
        dec.fold(stream=stream)
    fold_ms = timed(g_fold, pre=g_steps)
    D = dec.fold_depth(stream).cpu().tolist()
    assert D == [every - 1] * wd.R, D
    del g_steps, g_fold
    dec.close()

    s_b = 2 if wd.s0_dtype == "bf16" else 4
    e_b = 2 if wd.qkv_dtype == "bf16" else 4
    n_state = wd.R * wd.H * wd.d_v * wd.d_k
    planes = 1 if wd.s0_dtype == "bf16" else 2
    img = n_state * planes * 2 if kernel != L.ONELA_KERNEL_SIMT else 0
    rec = (every - 1) * wd.R * wd.H * (4 + 4 * wd.d_v + e_b * wd.d_k)
    fold_bytes = 2 * n_state * s_b + img + rec + wd.R * wd.W * (every - 1) * 4
    hbm = measured_peaks()[0]
    ach = fold_bytes / (fold_ms / 1e3) / 1e9
    out["fold"] = {"us": round(fold_ms * 1e3, 3), "launches": 1 if img else 2, "depth": every - 1,
                 "roofline": {"bound": "hbm", "achieved": round(ach, 1), "peak": hbm, "unit": "GB/s",
                              "frac": round(ach / hbm, 5), "alg_bytes": int(fold_bytes)}}
    return out


def time_sweep(device, stream, flush, reps=10, warmup=3):
    """The beam-width sweep (W = 64 .. 1024, T = 5, 1K-prompt shapes), the
    request sweep (R = 1, 8, 32 at H = 16, d = 128, W = 256, T = 7), the
    head sizes d = 64 and 256 at R = 1, H = 16, W = 256, T = 7, the headline
    shapes with a bf16 S0 and the op1k workload (T = 3): one whole
    decode (one onela_decode_steps call) per CUDA graph, L2 flushed before
    each, CUDA events; algorithmic bytes from the byte model.  S0 is drawn
    directly (its values do not change the work).  Returns the JSON object
    for the bench line."""
    import linear_attention_beam_shared_b200 as L
    cases = [synth.workload(f"wsweep{w}") for w in (64, 128, 256, 512, 1024)]
    cases += [synth.shape_sweep_workload(R, 16, 128, 256, 7) for R in (1, 8, 32)]
    cases += [synth.shape_sweep_workload(1, 16, d, 256, 7) for d in (64, 256)]
    cases += [synth.workload("long5k_bf16")]  # the headline shapes with a bf16 S0
    cases += [synth.workload("op1k")]         # the 1K-prompt workload: T = 3
    hbm = measured_peaks()[0]
    points = []
    for wl in cases:
        steps = synth.draw_decode(wl)
        S0 = synth.cast_state(0.1 * np.random.default_rng(wl.seed_id).standard_normal(
            (wl.R, wl.H, wl.d_v, wl.d_k)), wl.s0_dtype)
        ds = [{k: (v.to(device) if isinstance(v, torch.Tensor) else v) for k, v in st.items()} for st in steps]
        outs = [torch.empty((wl.R, st["W"], wl.H, wl.d_v), dtype=torch.float32, device=device) for st in steps]
        dec = L.BeamDecoder(wl.R, wl.H, wl.d_k, wl.d_v, wl.W, wl.T, wl.s0_dtype, wl.qkv_dtype,
                            device=device.index)
        dec.set_prompt_state(S0.to(device))
        g, launches, ev = decode_graph(dec, ds, outs, stream, flush=flush)
        kind = {L.ONELA_KERNEL_SIMT: "simt", L.ONELA_KERNEL_TC: "tc"}[dec.kernel]
        ms = time_graph(g, stream, flush, reps, warmup, ev=ev)
        del g
        assert dec.status() == 0
        dec.close()
        alg, _, _ = byte_model(wl, steps)
        gbs = alg / (ms / 1e3) / 1e9
        points.append({"workload": wl.name, "R": wl.R, "H": wl.H, "d": wl.d_k, "W": wl.W, "T": wl.T, "s0": wl.s0_dtype,
                       "kernel": kind,
                       "launches": launches, "ms_per_decode": round(ms, 5), "value": round(wl.units / (ms / 1e3), 1),
                       "achieved_gbs": round(gbs, 1), "frac": round(gbs / hbm, 4),
                       "capacity_ratio": capacity(wl)["ratio"]})
        del ds, outs
    return {"unit": UNIT, "peak_gbs": hbm, "l2": "flushed (512 MiB write) before every decode; decode timed by events inside its graph", "points": points}


def grid_inputs(R, H, d, W, T, device, seed):
    """Timing inputs for one shape of the multi-request grid, made on the
    device with the workload recipe (q, k unit-norm Gaussian, v Gaussian,
    alpha ~ U(0.85, 0.999) passed as log, beta = sigmoid(Gaussian), bf16
    q/k/v; parents uniform for even requests and truncated Zipf(1.1) over the
    previous beam rank for odd ones (Zipf when R = 1); S0 Gaussian 0.1).  The
    values do not change the work; the parents fix the ancestors replayed.
    Returns (S0, device steps, the same steps with CPU parents)."""
    g = torch.Generator(device=device).manual_seed(seed)
    S0 = 0.1 * torch.randn((R, H, d, d), generator=g, device=device)
    zipf = torch.tensor(synth.zipf_probs(W, 1.1), device=device, dtype=torch.float32)
    steps, cpu_steps = [], []
    for t in range(1, T + 1):
        q = torch.nn.functional.normalize(torch.randn((R, W, H, d), generator=g, device=device), dim=-1)
        k = torch.nn.functional.normalize(torch.randn((R, W, H, d), generator=g, device=device), dim=-1)
        v = torch.randn((R, W, H, d), generator=g, device=device)
        alpha = 0.85 + 0.149 * torch.rand((R, W, H), generator=g, device=device)
        beta = torch.sigmoid(torch.randn((R, W, H), generator=g, device=device))
        if t == 1:
            par = torch.zeros((R, W), dtype=torch.int32, device=device)
        else:
            rows = []
            for r in range(R):
                if R > 1 and r % 2 == 0:
                    rows.append(torch.randint(0, W, (W,), generator=g, device=device))
                else:
                    rows.append(torch.multinomial(zipf, W, replacement=True, generator=g))
            par = torch.stack(rows).to(torch.int32)
        st = {"q": q.to(torch.bfloat16), "k": k.to(torch.bfloat16), "v": v.to(torch.bfloat16),
              "g": torch.log(alpha).float(), "beta": beta.float(), "parents": par, "W": W, "W_prev": 1 if t == 1 else W}
        steps.append(st)
        cpu_steps.append({"parents": par.cpu(), "W": W})
    return S0, steps, cpu_steps


def time_grid(device, stream, flush, reps=3, warmup=1, full=True):
    """The multi-request operator-shape grid: R in {1, 8, 32}, H in {8, 16, 32},
    d_k = d_v in {64, 128, 256}, W in {128, 256, 512}, T in {1, 3, 5, 7} (fp32
    S0, bf16 q/k/v), each shape one onela_decode_steps call per CUDA graph, L2
    flushed before every decode.  full = False: R = 1 only.  Returns the JSON
    object for the bench line (a row per shape and a summary)."""
    import linear_attention_beam_shared_b200 as L
    hbm = measured_peaks()[0]
    rows, fracs = [], {}
    for R in ((1, 8, 32) if full else (1,)):
        for H in (8, 16, 32):
            for d in (64, 128, 256):
                for W in (128, 256, 512):
                    for T in (1, 3, 5, 7):
                        wl = synth.shape_sweep_workload(R, H, d, W, T)
                        free, _ = torch.cuda.mem_get_info(device)
                        need = (T * R * H * W * (4 + 4 * d + 2 * d) + T * R * W * H * d * (3 * 2 + 4)) * 1.3
                        if need > free * 0.8:
                            rows.append([R, H, d, W, T, None, None, "skipped: does not fit"])
                            continue
                        S0, ds, cpu_steps = grid_inputs(R, H, d, W, T, device, seed=R * 1000 + H * 37 + d + W + T)
                        outs = [torch.empty((R, W, H, d), dtype=torch.float32, device=device) for _ in ds]
                        dec = L.BeamDecoder(R, H, d, d, W, T, "f32", "bf16", device=device.index)
                        dec.set_prompt_state(S0)
                        g, launches, ev = decode_graph(dec, ds, outs, stream, flush=flush)
                        kind = {L.ONELA_KERNEL_SIMT: "simt", L.ONELA_KERNEL_TC: "tc"}[dec.kernel]
                        ms = time_graph(g, stream, flush, reps, warmup, ev=ev)
                        del g
                        assert dec.status() == 0
                        dec.close()
                        alg, _, _ = byte_model(wl, cpu_steps)
                        frac = alg / (ms / 1e3) / 1e9 / hbm
                        fracs.setdefault(kind, []).append(frac)
                        rows.append([R, H, d, W, T, round(ms, 5), round(frac, 4), kind])
                        del ds, outs, S0
                        torch.cuda.empty_cache()
    allf = sorted(f for v in fracs.values() for f in v)
    summary = {"shapes": len(rows), "timed": len(allf),
               "median_frac": round(statistics.median(allf), 4) if allf else None,
               "worst_frac": round(allf[0], 4) if allf else None, "best_frac": round(allf[-1], 4) if allf else None,
               "by_kernel": {k: {"shapes": len(v), "median_frac": round(statistics.median(v), 4),
                                 "worst_frac": round(min(v), 4)} for k, v in fracs.items()}}
    return {"unit": "fraction of measured HBM bandwidth (algorithmic bytes)", "peak_gbs": hbm,
            "l2": "flushed before every decode", "columns": ["R", "H", "d", "W", "T", "ms_per_decode", "frac", "kernel"],
            "summary": summary, "rows": rows}


def decode_graph(dec, dsteps, outs, stream, per_step=False, flush=None):
    """One whole decode through the public API captured in a CUDA graph: one
    onela_decode_steps call, or (per_step) one onela_decode_step call per
    step.  With flush: the graph is [512 MiB write that flushes L2] [start
    event] [the decode] [end event], so that the events time the decode's
    kernels on the device and not the launch of the graph.  Returns (graph,
    kernel launches per decode, (start, end) events or None)."""
    def run():
        if per_step:
            for st, o in zip(dsteps, outs):
                dec.step(st["q"], st["k"], st["v"], st["g"], st["beta"], st["parents"], o=o, stream=stream)
        else:
            dec.steps(dsteps, outs, stream=stream)
    with torch.cuda.stream(stream):
        run()
    stream.synchronize()
    assert dec.status() == 0
    launches = len(dsteps) if per_step else dec.last_launches()
    dec.reset(stream)
    graph = torch.cuda.CUDAGraph()
    ev = None
    with torch.cuda.graph(graph, stream=stream):
        if flush is not None:
            # External events: real event-record nodes in the graph (not the
            # capture's internal dependencies), readable after each replay.
            ev = (torch.cuda.Event(enable_timing=True, external=True),
                  torch.cuda.Event(enable_timing=True, external=True))
            flush.fill_(1)
            ev[0].record(stream)
        run()
        if flush is not None:
            ev[1].record(stream)
    dec.reset(stream)
    return graph, launches, ev


def time_graph(graph, stream, flush, reps, warmup, ev=None):
    """Mean device time (ms, max over ranks) of a decode.  ev given (a graph
    from decode_graph with flush): each replay writes 512 MiB and times the
    decode between its own events.  Otherwise each replay follows a 512 MiB
    write and is timed from outside, graph launch included."""
    with torch.cuda.stream(stream):
        for _ in range(warmup):
            if ev is None:
                flush.fill_(9)
            graph.replay()
    stream.synchronize()
    total = 0.0
    if ev is not None:
        for _ in range(reps):
            with torch.cuda.stream(stream):
                graph.replay()
            stream.synchronize()
            total += ev[0].elapsed_time(ev[1])
        return max_over_ranks(total / reps, stream.device)
    evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(reps)]
    with torch.cuda.stream(stream):
        for i, (e0, e1) in enumerate(evs):
            flush.fill_(i & 0xFF)
            e0.record(stream)
            graph.replay()
            e1.record(stream)
    stream.synchronize()
    return max_over_ranks(sum(e0.elapsed_time(e1) for e0, e1 in evs) / reps, stream.device)


def byte_model(wl, steps):
    """Algorithmic bytes of one whole decode (all T steps): every byte the
    method must move at least once, with each distinct ancestor record counted
    once; plus the per-beam-gather upper bound."""
    s = 2 if wl.s0_dtype == "bf16" else 4
    e = 2 if wl.qkv_dtype == "bf16" else 4
    d_k, d_v, H, R = wl.d_k, wl.d_v, wl.H, wl.R
    rec = 4 + 4 * d_v + e * d_k
    total = upper = 0
    per_step = []
    for t, st in enumerate(steps, start=1):
        W = st["W"]
        plist = [x["parents"].numpy() for x in steps[:t]]
        U = [synth.distinct_ancestors([p[r] for p in plist], t) for r in range(R)]
        base = R * H * (d_k * d_v * s + W * ((2 * d_k + d_v) * e + 8) + W * (4 * d_v + 4 * d_v + 4 + d_k * e))
        idx = R * (W * 4 + W * (t - 1) * 4)
        b_t = base + idx + H * sum(U) * rec
        u_t = base + idx + H * R * W * (t - 1) * rec
        per_step.append(b_t)
        total += b_t
        upper += u_t
    return total, upper, per_step


def capacity(wl):
    """State memory per (request, head) at the end of a T-step decode: this
    library's (S0 in its dtype, the T depths of records (alpha fp32, delta fp32,
    k in the q/k/v dtype), the ancestry rows and parents shared by the
    request's heads) against a full-state beam decode that keeps one fp32
    d_v x d_k state per beam (the pages' FullState)."""
    s = 2 if wl.s0_dtype == "bf16" else 4
    e = 2 if wl.qkv_dtype == "bf16" else 4
    T, W, dk, dv, H = wl.T, wl.W, wl.d_k, wl.d_v, wl.H
    onela = dk * dv * s + T * W * (4 + 4 * dv + e * dk) + T * W * (T + 1) * 4 / H
    full = W * dk * dv * 4
    return {"bytes_per_request_head": int(round(onela)), "fullstate_fp32_bytes_per_request_head": int(full),
            "ratio": round(full / onela, 2)}


class ClockSampler:
    """nvidia-smi samples during the timed region."""

    def __init__(self, gpu_index):
        self.proc = None
        self.gpu = gpu_index
        # The raw samples go to ONELA_CLOCKS_CSV when set, else a temporary file.
        self.path = os.environ.get("ONELA_CLOCKS_CSV") or os.path.join(
            tempfile.gettempdir(), f"onela_clocks_{os.getpid()}_{gpu_index}.csv")

    def __enter__(self):
        q = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
             "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
             "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")
        try:
            self.f = open(self.path, "w")
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--query-gpu={q}", "--format=csv,noheader,nounits", "-lms", "100",
                 "-i", str(self.gpu)], stdout=self.f, stderr=subprocess.DEVNULL)
        except Exception:
            self.proc = None
        time.sleep(0.3)
        return self

    def __exit__(self, *a):
        if self.proc is not None:
            time.sleep(0.2)
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except Exception:
                self.proc.kill()
            self.f.close()

    def summary(self):
        if self.proc is None or not os.path.exists(self.path):
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        rows = []
        with open(self.path) as f:
            for line in f:
                parts = [x.strip() for x in line.split(",")]
                if len(parts) >= 9:
                    rows.append(parts)
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["no samples"]}
        sm = [float(r[1]) for r in rows if r[1].replace(".", "").isdigit()]
        mx = [float(r[2]) for r in rows if r[2].replace(".", "").isdigit()]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in rows for i in range(4) if r[5 + i].lower().startswith("active")})
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": max(mx) if mx else None,
                "reasons": reasons, "samples": len(rows)}


def time_cpu_oracle(wl, S0, steps, budget_s=10.0, nthreads=0):
    """The C fp64 full-state oracle as it stands, on the host cores.  Runs the
    whole decode repeatedly until about budget_s of CPU work is done."""
    from oracle import cref
    cref.beam_decode_fullstate(S0[:, :1], [{k: (v[:, :, :1] if k in ("q", "k", "v", "g", "beta") else v)
                                            for k, v in s.items()} for s in steps[:1]], nthreads=nthreads)
    reps, t0 = 0, time.perf_counter()
    while True:
        cref.beam_decode_fullstate(S0, steps, nthreads=nthreads)
        reps += 1
        el = time.perf_counter() - t0
        if el >= budget_s or reps >= 1000:
            break
    units = wl.units * reps
    threads = nthreads if nthreads > 0 else cref.max_threads()
    return units / el, reps, el, threads


# ---------------------------------------------------------------- our arm
def run_ours(args):
    ws, rank, local = dist_env()
    if ws > 1:
        import torch.distributed as dist
        from datetime import timedelta
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=timedelta(seconds=120),
                                device_id=torch.device("cuda", local))
    else:
        torch.cuda.set_device(0)
    device = torch.device("cuda", torch.cuda.current_device())
    import linear_attention_beam_shared_b200 as L

    wl = rank_workload(synth.workload(args.workload), rank)
    if args.s0 == "prefill":
        S0 = s0_by_prefill_gpu(wl, device)
    else:   # same shapes and dtype, entries drawn directly (for quick profiling runs)
        S0 = synth.cast_state(0.1 * np.random.default_rng(wl.seed_id).standard_normal(
            (wl.R, wl.H, wl.d_v, wl.d_k)), wl.s0_dtype)
    steps = synth.draw_decode(wl)
    kernel = {"auto": L.ONELA_KERNEL_AUTO, "simt": L.ONELA_KERNEL_SIMT, "tc": L.ONELA_KERNEL_TC}[args.kernel]
    # One whole decode = one onela_decode_steps call with every step's inputs
    # resident (each step after the first overlaps the one before it; no
    # handle flag and no contract across calls).
    dec = L.BeamDecoder(wl.R, wl.H, wl.d_k, wl.d_v, wl.W, wl.T, wl.s0_dtype, wl.qkv_dtype,
                        kernel=kernel, device=device.index)
    dec.set_prompt_state(S0.to(device))
    dsteps = [{k: (v.to(device) if isinstance(v, torch.Tensor) else v) for k, v in s.items()} for s in steps]
    outs = [torch.empty((wl.R, s["W"], wl.H, wl.d_v), dtype=torch.float32, device=device) for s in steps]

    stream = torch.cuda.Stream(device=device)
    flush = torch.empty(512 * 1024 * 1024, dtype=torch.uint8, device=device)
    # Eager warm-up of the API (also loads the module), then capture: each
    # replay writes 512 MiB (flushing L2), then the decode runs between two
    # events recorded inside the graph.
    graph, launches, ev = decode_graph(dec, dsteps, outs, stream, flush=flush)
    kind = {L.ONELA_KERNEL_SIMT: "simt", L.ONELA_KERNEL_TC: "tc"}[dec.kernel]
    with torch.cuda.stream(stream):
        for _ in range(args.warmup):
            graph.replay()
    stream.synchronize()

    if ws > 1:
        torch.distributed.barrier()
    torch.cuda.synchronize()
    times_ms = []
    with ClockSampler(device.index) as clk:
        for i in range(args.steps):
            with torch.cuda.stream(stream):
                graph.replay()
            stream.synchronize()
            times_ms.append(ev[0].elapsed_time(ev[1]))
        torch.cuda.synchronize()
    if ws > 1:
        torch.distributed.barrier()
    total_ms = max_over_ranks(sum(times_ms), device)
    assert dec.status() == 0
    ms_per_step = total_ms / args.steps
    value = whole_job_value(wl.units, ws, ms_per_step)
    del graph
    # The same decode timed from outside its graph (graph launch included).
    graph2, _, _ = decode_graph(dec, dsteps, outs, stream)
    ms_incl_launch = time_graph(graph2, stream, flush, reps=min(args.steps, 50), warmup=3)
    del graph2
    dec.close()

    # Roofline of the decode kernel (the only kernel in the step).
    alg_bytes, upper_bytes, _ = byte_model(wl, steps)
    hbm, bf16_tf, bf16_sus, src = measured_peaks()
    achieved = alg_bytes / launches / (ms_per_step / launches / 1e3) / 1e9
    traffic = ncu_traffic(kind)
    roofline = {
        "bound": "hbm", "achieved": round(achieved, 1), "peak": hbm, "unit": "GB/s",
        "frac": round(achieved / hbm, 4),
        "traffic": traffic["bytes_per_launch"] if traffic else None,
        "peak_source": f"{src} (MEASURED_PEAKS.json hbm_gbs)" if src == "measured" else "fallback",
        "kernel": {"tc": "tensor-core step kernel", "simt": "SIMT step kernel"}[kind],
        "launches_per_decode": launches,
        "alg_bytes_per_launch": round(alg_bytes / launches),
        "upper_bound_bytes_per_launch": round(upper_bytes / launches),
        "avg_launch_us": round(ms_per_step * 1e3 / launches, 3),
    }
    flops = 4 * wl.d_k * wl.d_v * wl.W * wl.H * wl.R * wl.T
    roofline["tensor_frac_of_sustained_bf16"] = round(flops / (ms_per_step / 1e3) / 1e12 / bf16_sus, 5) if bf16_sus else None

    # The same decode as one onela_decode_step call per step: under
    # ONELA_FLAG_PDL (steps overlap by its contract across calls), and with
    # ordinary launches (each step waits for the one before it).
    variants = None
    if not args.no_variants and kind == "tc":
        variants = {}
        for name, fl in (("per_step_calls_pdl_flag", L.ONELA_FLAG_PDL), ("per_step_calls", 0)):
            d2 = L.BeamDecoder(wl.R, wl.H, wl.d_k, wl.d_v, wl.W, wl.T, wl.s0_dtype, wl.qkv_dtype,
                               kernel=kernel, device=device.index, flags=fl)
            d2.set_prompt_state(S0.to(device))
            g2, n2, ev2 = decode_graph(d2, dsteps, outs, stream, per_step=True, flush=flush)
            ms2 = time_graph(g2, stream, flush, reps=20, warmup=3, ev=ev2)
            del g2
            assert d2.status() == 0
            d2.close()
            variants[name] = {"ms_per_decode": round(ms2, 5), "launches": n2,
                              "frac": round(alg_bytes / (ms2 / 1e3) / 1e9 / hbm, 4)}

    # End to end through the public API with host buffers: per step the H2D
    # copy of that step's inputs from pinned memory, the decode call, and the
    # D2H read of its output o.  Each step's inputs travel as one packed copy
    # on an upload stream, the step waits for its own copy on the compute
    # stream, and its o returns on a download stream, so uploads, steps and
    # downloads of different steps overlap (the two copy directions run on
    # separate engines).  A handle without the programmatic-launch flag: a
    # copy, not the previous step, is what each step waits for.
    dec = L.BeamDecoder(wl.R, wl.H, wl.d_k, wl.d_v, wl.W, wl.T, wl.s0_dtype, wl.qkv_dtype,
                        kernel=kernel, device=device.index)
    dec.set_prompt_state(S0.to(device))
    keys = ("q", "k", "v", "g", "beta", "parents")
    host_pack, dev_pack, dev_views = [], [], []
    for st in steps:
        offs, n = [], 0
        for key in keys:
            offs.append(n)
            n = (n + st[key].numel() * st[key].element_size() + 255) & ~255
        hb = torch.empty(n, dtype=torch.uint8).pin_memory()
        for key, off in zip(keys, offs):
            b = st[key].contiguous().view(-1).view(torch.uint8)
            hb[off:off + b.numel()].copy_(b)
        db = torch.empty(n, dtype=torch.uint8, device=device)
        dev_views.append({key: db[off:off + st[key].numel() * st[key].element_size()].view(st[key].dtype)
                          .view(st[key].shape) for key, off in zip(keys, offs)})
        host_pack.append(hb)
        dev_pack.append(db)
    host_out = [torch.empty(o.shape, dtype=o.dtype).pin_memory() for o in outs]
    h2d = sum(st[key].numel() * st[key].element_size() for st in steps for key in keys)
    d2h = sum(o.numel() * o.element_size() for o in outs)
    s_up = torch.cuda.Stream(device=device)
    s_down = torch.cuda.Stream(device=device)
    ev_in = [torch.cuda.Event() for _ in steps]
    ev_o = [torch.cuda.Event() for _ in steps]
    e_start = torch.cuda.Event(enable_timing=True)
    e_end = torch.cuda.Event(enable_timing=True)
    e2e_steps = max(1, min(args.steps, 20))

    def enqueue_e2e():
        s_up.wait_stream(stream)
        s_down.wait_stream(stream)
        with torch.cuda.stream(s_up):
            for hb, db, ev in zip(host_pack, dev_pack, ev_in):
                db.copy_(hb, non_blocking=True)
                ev.record(s_up)
        for ds, o, ho, ei, eo in zip(dev_views, outs, host_out, ev_in, ev_o):
            stream.wait_event(ei)
            dec.step(ds["q"], ds["k"], ds["v"], ds["g"], ds["beta"], ds["parents"], o=o, stream=stream)
            eo.record(stream)
            s_down.wait_event(eo)
            with torch.cuda.stream(s_down):
                ho.copy_(o, non_blocking=True)
        stream.wait_stream(s_down)

    # (1) issued from the host, call by call, inside the timed region.
    e2e_eager_ms = 0.0
    for it in range(e2e_steps + 1):
        with torch.cuda.stream(stream):
            flush.fill_(3)
            dec.reset(stream)
            e_start.record(stream)
        enqueue_e2e()
        e_end.record(stream)
        stream.synchronize()
        if it > 0:
            e2e_eager_ms += e_start.elapsed_time(e_end)
    for o, ho in zip(outs, host_out):
        assert torch.equal(o.cpu(), ho), "downloaded output differs from the device copy"
    eager_out = [ho.clone() for ho in host_out]
    # (2) the same copies and calls captured in one CUDA graph (the uploads,
    # the steps and the downloads on their three streams), replayed: no host
    # work inside the timed region, every byte still crosses PCIe each step.
    dec.reset(stream)
    g_e2e = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g_e2e, stream=stream):
        enqueue_e2e()
    dec.reset(stream)
    for o, ho in zip(outs, host_out):
        o.zero_()
        ho.zero_()
    e2e_ms = 0.0
    for it in range(e2e_steps + 1):
        with torch.cuda.stream(stream):
            flush.fill_(3)
            e_start.record(stream)
            g_e2e.replay()
            e_end.record(stream)
        stream.synchronize()
        if it > 0:
            e2e_ms += e_start.elapsed_time(e_end)
    del g_e2e
    for o, ho, eo in zip(outs, host_out, eager_out):
        assert torch.equal(o.cpu(), ho), "downloaded output differs from the device copy"
        assert torch.equal(ho, eo), "graph replay differs from the calls issued one by one"
    e2e_ms = max_over_ranks(e2e_ms, device)
    e2e_eager_ms = max_over_ranks(e2e_eager_ms, device)
    e2e = {"value": round(whole_job_value(wl.units, ws, e2e_ms / e2e_steps), 1), "unit": UNIT,
           "copies": "one packed pinned H2D per step on an upload stream, the step, D2H of o on a download "
                     "stream, uploads, steps and downloads overlapping; captured in one CUDA graph per decode",
           "h2d_bytes_per_step": int(h2d), "d2h_bytes_per_step": int(d2h),
           "issued_call_by_call": round(whole_job_value(wl.units, ws, e2e_eager_ms / e2e_steps), 1)}
    assert dec.status() == 0

    prefill = time_prefill(wl, device, stream, flush) if (wl.L_prompt > 0 and not args.no_prefill) else None
    select = None if args.no_prefill else time_select(device, stream, flush, R=wl.R, W_prev=wl.W, C=256, W=wl.W)
    sweep = None if (args.no_sweep or ws > 1) else time_sweep(device, stream, flush)
    grid = None if (args.no_grid or ws > 1) else time_grid(device, stream, flush, full=not args.grid_r1)
    fold = None if args.no_prefill else [time_fold(wl, S0, kernel, device, stream, flush, every=4),
                                          time_fold(wl, S0, kernel, device, stream, flush, every=8, alone=False),
                                          time_fold(wl, S0, kernel, device, stream, flush, T=32, every=8, alone=False,
                                                    tmax=16)]

    cpu = None
    if rank == 0 and ws == 1 and not args.no_cpu:
        rate, reps, el, threads = time_cpu_oracle(wl, S0, steps, budget_s=args.cpu_budget)
        cpu = {"value": round(rate, 1), "unit": UNIT, "cores": threads, "kind": "oracle",
               "sample": f"whole {args.workload} decode (R=1,H={wl.H},W={wl.W},T={wl.T}) x{reps} "
                         f"in {el:.1f} s, plain-C fp64 full-state oracle"}

    dec.close()
    if rank == 0:
        line = {
            "metric": METRIC, "value": round(value, 1), "unit": UNIT, "n_gpus": ws,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(ms_per_step, 6),
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f32",
            "data": "synthetic",
            "config": {"workload": f"{args.workload}: R={wl.R} per GPU, H={wl.H}, d_k=d_v={wl.d_k}, "
                                   f"W={wl.W}, T={wl.T}, L_prompt={wl.L_prompt}, S0 {wl.s0_dtype}, "
                                   f"q/k/v {wl.qkv_dtype}, parents Zipf(1.1)",
                       "global_batch": wl.R * ws, "seq_len": wl.T, "parallelism": f"replicas{ws}",
                       "l2": "flushed (512 MiB write inside the graph, before the start event) before every timed step", "kernel": kind,
                       "step": f"one whole {wl.T}-step decode (one onela_decode_steps call) in a CUDA graph",
                       "launches_per_decode": launches},
            "roofline": roofline, "cpu_baseline": cpu, "e2e": e2e,
            "clocks": clk.summary(), "gpu_launches": launches * args.steps,
            "variants": variants, "capacity": capacity(wl),
            "ms_per_step_graph_launch_included": round(ms_incl_launch, 6),
            "prefill": prefill, "beam_select": select, "fold": fold, "sweep": sweep, "grid": grid,
        }
        print(json.dumps(line))
    if ws > 1:
        torch.distributed.destroy_process_group()


# ---------------------------------------------------------- reference arm
def run_reference(args):
    ws, rank, _ = dist_env()
    if rank != 0:
        return
    from oracle import cref
    wl = synth.workload(args.workload)
    # S0 values do not change the oracle's running time; draw them directly
    # instead of running a long prefill on the host.
    S0 = synth.cast_state(0.1 * np.random.default_rng(0).standard_normal((wl.R, wl.H, wl.d_v, wl.d_k)),
                          wl.s0_dtype)
    steps = synth.draw_decode(wl)
    for _ in range(args.warmup):
        cref.beam_decode_fullstate(S0, steps)
    t0 = time.perf_counter()
    for _ in range(args.steps):
        cref.beam_decode_fullstate(S0, steps)
    el = time.perf_counter() - t0
    value = wl.units * args.steps / el
    threads = cref.max_threads()
    line = {
        "impl": "reference", "metric": METRIC, "value": round(value, 1), "unit": UNIT, "n_gpus": ws,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(el / args.steps * 1e3, 3),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic",
        "config": {"workload": f"{args.workload}: R={wl.R}, H={wl.H}, d_k=d_v={wl.d_k}, W={wl.W}, "
                               f"T={wl.T}", "global_batch": wl.R, "seq_len": wl.T,
                   "parallelism": "host cores"},
        "cpu_baseline": {"value": round(value, 1), "unit": UNIT, "cores": threads, "kind": "oracle",
                         "sample": f"whole {args.workload} decode per step, plain-C fp64 full-state oracle"},
        "e2e": {"value": round(value, 1), "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line))


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=2000)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", default="long5k")
    ap.add_argument("--kernel", choices=["auto", "simt", "tc"], default="auto")
    ap.add_argument("--no-cpu", action="store_true", help="skip the CPU-oracle baseline leg")
    ap.add_argument("--no-variants", action="store_true",
                    help="skip timing the one-launch-per-step variants of the headline decode")
    ap.add_argument("--cpu-budget", type=float, default=10.0)
    ap.add_argument("--no-prefill", action="store_true", help="skip the prefill, beam-selection and fold timings")
    ap.add_argument("--no-sweep", action="store_true", help="skip the beam-width and request sweeps")
    ap.add_argument("--no-grid", action="store_true", help="skip the multi-request shape grid")
    ap.add_argument("--grid-r1", action="store_true", help="the shape grid at R = 1 only (the default runs R = 1, 8, 32)")
    ap.add_argument("--s0", choices=["prefill", "direct"], default="prefill",
                    help="S0 from the GDN recurrence over the synthetic prompt (default) or drawn "
                         "directly; the decode's work does not depend on the S0 values")
    args = ap.parse_args()
    if args.warmup < 3 and args.impl == "ours":
        args.warmup = 3
    if args.impl == "reference":
        run_reference(args)
    else:
        run_ours(args)


if __name__ == "__main__":
    main()
