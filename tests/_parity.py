"""Shared helpers for the GPU-vs-oracle parity tests.

Inputs come from the seeded generator; expected values come from the CPU
oracle only. The CUDA path is reached through the ctypes binding.
"""
from __future__ import annotations

import math

import numpy as np
import torch

from oracle import dhsa as ora
from long_context_prefill_dhsa_b200 import inputs as I

MAX_ABS = 2e-2     # bf16 output vs fp32/fp64 oracle, per element
MEAN_ABS = 2e-3    # averaged over the compared elements
POOL_RTOL = 2e-5   # fp32 accumulation of <= 1024 bf16 rows vs fp64
NEAR_TIE_REL = 1e-5


def to_dev(d, device="cuda"):
    f = lambda a: torch.from_numpy(np.ascontiguousarray(a)).to(device)
    return dict(Q=f(d["Q"]).view(torch.bfloat16), K=f(d["K"]).view(torch.bfloat16),
                V=f(d["V"]).view(torch.bfloat16), off=f(d["off"]), n_chunks=f(d["n_chunks"]))


def gpu_sel_rows(sel, n_sel):
    """GPU sel tensor -> nested python lists like the oracle's (rows with n_sel > 0)."""
    sel = sel.cpu().numpy()
    n_sel = n_sel.cpu().numpy()
    B, Hq, nmax, _ = sel.shape
    return [[[sel[b, h, i, :n_sel[b, h, i]].astype(np.int64) for i in range(nmax) if n_sel[b, h, i] > 0]
             for h in range(Hq)] for b in range(B)]


def compare_selection(S, sel_ora, sel_gpu, n_chunks, k):
    """Exact per-row equality except oracle near-tie rows; a mismatched
    near-tie row must still be a valid top-k under a tolerance band.
    Returns (n_rows, n_near_tie_mismatch)."""
    rows = mism = 0
    for b in range(len(sel_ora)):
        for h in range(len(sel_ora[b])):
            for i in range(int(n_chunks[b])):
                rows += 1
                a, g = sel_ora[b][h][i], sel_gpu[b][h][i]
                if len(a) == len(g) and np.array_equal(a, g):
                    continue
                Srow = S[b, h, i]
                assert ora.near_tie(Srow, i, k, NEAR_TIE_REL), \
                    f"selection mismatch outside near-tie band at b={b} h={h} i={i}: {a} vs {g}"
                assert len(g) == len(a) and g[-1] == i and np.all(np.diff(g) > 0)
                scale = float(np.max(np.abs(Srow[:i])))
                kth = np.sort(Srow[:i])[::-1][k - 1]
                assert np.min(Srow[g[:-1]]) >= kth - NEAR_TIE_REL * scale
                mism += 1
    return rows, mism


def compare_out(O_gpu, O_ref, mask=None):
    """max-abs / mean-abs between bf16 GPU output and the oracle."""
    og = O_gpu.float().cpu().numpy().astype(np.float64)
    if mask is not None:
        og, ref = og[mask], O_ref[mask]
    else:
        ref = O_ref
    assert np.all(np.isfinite(og)), "non-finite GPU output"
    err = np.abs(og - ref)
    return float(err.max()), float(err.mean())


def oracle_full(d, k, attn_dtype=np.float64, rows=None):
    """Oracle routing (fp64) + attention for a (small) workload dict."""
    Q, K, V = ora.bf16_to_f64(d["Q"]), ora.bf16_to_f64(d["K"]), ora.bf16_to_f64(d["V"])
    Qp, Kp, S, sel = ora.routing(Q, K, d["off"], d["n_chunks"], k)
    return Q, K, V, Qp, Kp, S, sel


def scale():
    return 1.0 / math.sqrt(128)
