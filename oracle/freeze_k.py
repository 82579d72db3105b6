"""Find k for the density-targeted workloads with the CPU oracle only.

For a workload with a target kept density, k is the smallest number of
earlier chunks per query chunk whose kept density -- kept token pairs over
causal pairs L(L+1)/2, averaged over (b, hq) -- reaches the target on the
seeded inputs. Prints one line per workload; the values are frozen into the
workload table of the package's inputs module and re-checked by the tests.

    python -m oracle.freeze_k [workload ...]
"""
from __future__ import annotations

import sys

import numpy as np

from oracle import dhsa


def pooled_scores(w, inputs_mod):
    """Oracle scores S[B,Hq,Nmax,Nmax] for workload w, one head at a time."""
    off, n_chunks = inputs_mod.offsets(w)
    nmax = off.shape[1] - 1
    Qp = np.zeros((w.B, w.Hq, nmax, 128))
    Kp = np.zeros((w.B, w.Hkv, nmax, 128))
    for hkv in range(w.Hkv):
        heads_q = list(range(hkv * w.G, (hkv + 1) * w.G))
        d = inputs_mod.make_inputs(w, heads_q=heads_q, heads_kv=[hkv], with_v=False)
        for hq in heads_q:
            Qp[:, hq:hq + 1] = dhsa.chunk_pool(dhsa.bf16_to_f64(d["Q"][:, hq:hq + 1]), off, n_chunks, nmax)
        Kp[:, hkv:hkv + 1] = dhsa.chunk_pool(dhsa.bf16_to_f64(d["K"][:, hkv:hkv + 1]), off, n_chunks, nmax)
        del d
    return off, n_chunks, dhsa.chunk_scores(Qp, Kp, n_chunks)


def density_for_k(S, off, n_chunks, k, L):
    return dhsa.density(off, n_chunks, dhsa.select(S, n_chunks, k), L)


def freeze(w, inputs_mod):
    off, n_chunks, S = pooled_scores(w, inputs_mod)
    lo, hi = 0, int(n_chunks.max())
    while lo < hi:                      # density grows with k
        mid = (lo + hi) // 2
        if density_for_k(S, off, n_chunks, mid, w.L) >= w.target_density:
            hi = mid
        else:
            lo = mid + 1
    return lo, density_for_k(S, off, n_chunks, lo, w.L)


def main(argv):
    from long_context_prefill_dhsa_b200 import inputs as inputs_mod
    names = argv or [n for n, w in inputs_mod.WORKLOADS.items() if w.target_density]
    for n in names:
        w = inputs_mod.WORKLOADS[n]
        k, dens = freeze(w, inputs_mod)
        print(f"{n}: target {w.target_density} -> k={k} density={dens:.4f}", flush=True)


if __name__ == "__main__":
    main(sys.argv[1:])
