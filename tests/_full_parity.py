"""Worker of the full-mode parity test (tests/test_gpu_full_parity.py).

One call checks one (batch element, kv head) group against the CPU oracle:
every pooled vector of the group's query heads and of its kv head, every
selection row of those query heads (exact, except rows the oracle flags as
near-ties, which are counted), and every output element, recomputed by the
oracle's fp32 attention over the GPU's selection. It runs in a spawned
worker process with one BLAS thread, so groups run in parallel; it imports
the oracle and numpy only (no CUDA).
"""
from __future__ import annotations

import math

import numpy as np

from oracle import dhsa as ora

MAX_ABS, MEAN_ABS, POOL_RTOL, NEAR_TIE_REL = 2e-2, 2e-3, 2e-5, 1e-5


def bf16_bits_of(x) -> np.ndarray:
    return np.ascontiguousarray(x).view(np.uint16)


def check_group(task: dict) -> dict:
    """task: b, hkv, hqs (query heads), k, off_b [Nmax+1], n (chunks), Q [G,L,128]
    (bf16 bits), K, V [L,128] (bf16 bits), O [G,L,128] (GPU output, bf16 bits),
    Qp_g [G,Nmax,128], Kp_g [Nmax,128] (GPU pooled, fp32), sel_g (list per query
    head of the GPU's kept chunks per row), needles [(hq, i, j)]."""
    off_b = task["off_b"][None, :]
    nc = np.array([task["n"]], dtype=np.int32)
    nmax = off_b.shape[1] - 1
    k = task["k"]
    K64 = ora.bf16_to_f64(task["K"])
    Kp = ora.chunk_pool(K64[None, None], off_b, nc, nmax)
    pool_bad = int(np.sum(np.abs(task["Kp_g"] - Kp[0, 0]) > POOL_RTOL * (np.abs(Kp[0, 0]) + 1.0)))
    Kf = K64.astype(np.float32)
    Vf = ora.bf16_to_f64(task["V"]).astype(np.float32)
    scale = 1.0 / math.sqrt(128)
    rows = near_tie_swaps = sel_bad = 0
    err_max, err_sum, err_n = 0.0, 0.0, 0
    for gi, hq in enumerate(task["hqs"]):
        Q64 = ora.bf16_to_f64(task["Q"][gi])
        Qp = ora.chunk_pool(Q64[None, None], off_b, nc, nmax)
        pool_bad += int(np.sum(np.abs(task["Qp_g"][gi] - Qp[0, 0]) > POOL_RTOL * (np.abs(Qp[0, 0]) + 1.0)))
        S = ora.chunk_scores(Qp, Kp, nc)
        sel_o = ora.select(S, nc, k)[0][0]
        sel_g = task["sel_g"][gi]
        for i in range(task["n"]):
            rows += 1
            a, g = sel_o[i], sel_g[i]
            if len(a) == len(g) and np.array_equal(a, g):
                continue
            Srow = S[0, 0, i]
            ok = ora.near_tie(Srow, i, k, NEAR_TIE_REL) and len(g) == len(a) and g[-1] == i and np.all(np.diff(g) > 0)
            if ok:
                scale_s = float(np.max(np.abs(Srow[:i])))
                kth = np.sort(Srow[:i])[::-1][k - 1]
                ok = np.min(Srow[g[:-1]]) >= kth - NEAR_TIE_REL * scale_s
            if ok:
                near_tie_swaps += 1
            else:
                sel_bad += 1
        Qf = Q64.astype(np.float32)
        Og = ora.bf16_to_f64(task["O"][gi])
        for i in range(task["n"]):
            s, e = int(off_b[0, i]), int(off_b[0, i + 1])
            ref = ora.attn_chunk(Qf, Kf, Vf, off_b[0], sel_g[i], i, scale, np.float32)
            err = np.abs(Og[s:e] - ref)
            err_max = max(err_max, float(err.max()))
            err_sum += float(err.sum())
            err_n += err.size
    needles_missed = sum(1 for (hq, i, j) in task["needles"] if hq in task["hqs"]
                         and j not in task["sel_g"][task["hqs"].index(hq)][i])
    return dict(b=task["b"], hkv=task["hkv"], rows=rows, near_tie_swaps=near_tie_swaps, sel_bad=sel_bad,
                pool_bad=pool_bad, err_max=err_max, err_sum=err_sum, err_n=err_n, needles_missed=needles_missed)
