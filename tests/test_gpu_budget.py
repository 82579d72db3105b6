"""GPU parity of the token-budget selection (include/dhsa.h, 2') against the
CPU oracle, through the C ABI, plus attention over the budget CSR.

Bars as in test_gpu_parity.py: selected chunk sets identical except rows the
oracle flags as near-ties anywhere in the ranked prefix the rule inspects
(gap below 1e-5 of the row's largest |score|); CSR bit-exact from the GPU's
own selection; attention max-abs <= 2e-2, mean-abs <= 2e-3.
"""
import numpy as np
import pytest
import torch

from oracle import dhsa as ora
from long_context_prefill_dhsa_b200 import inputs as I
from tests import _parity as P

pytestmark = pytest.mark.gpu

needs_gpu = pytest.mark.skipif(not torch.cuda.is_available(), reason="needs a CUDA device")


@pytest.fixture(scope="module")
def lib():
    from long_context_prefill_dhsa_b200 import binding
    return binding


def _compare_budget(S, off, nc, sel_gpu, budget, recent, k_max, heads=None):
    """Exact per-row equality except near-tie rows; returns (rows, near-tie mismatches)."""
    rows = mism = 0
    B = len(sel_gpu)
    for b in range(B):
        n = int(nc[b])
        lens = np.diff(off[b, : n + 1])
        for hi in range(S.shape[1]):
            hq = hi if heads is None else heads[hi]
            for i in range(n):
                bud = int(budget if np.isscalar(budget) else budget[b, hq, i])
                want = ora.select_budget_row(S[b, hi, i], lens, i, bud, recent, k_max)
                got = sel_gpu[b][hi][i]
                rows += 1
                if len(got) == len(want) and np.array_equal(got, want):
                    continue
                assert ora.budget_near_tie(S[b, hi, i], lens, i, bud, recent, k_max, P.NEAR_TIE_REL), \
                    f"budget selection mismatch at b={b} hq={hq} i={i}: oracle {want} gpu {got}"
                assert got[-1] == i and np.all(np.diff(got) > 0) and len(got) <= k_max + 1
                mism += 1
    return rows, mism


CASES = [
    # name, workload, budget, recent, k_max
    ("tiny-b60-r0", I.WORKLOADS["tiny"], 60, 0, 8),
    ("tiny-b200-r2", I.WORKLOADS["tiny"], 200, 2, 8),
    ("long-chunks", I.custom(B=1, Hq=4, Hkv=1, L=1500, lo=100, hi=700, k=2, wid=102), 900, 1, 4),
    ("batch2-gqa8", I.custom(B=2, Hq=8, Hkv=1, L=777, lo=3, hi=90, k=4, wid=103), 150, 1, 12),
    ("budget0-window", I.custom(B=1, Hq=2, Hkv=1, L=1000, lo=1, hi=300, k=0, wid=104), 0, 3, 6),
    ("kmax0", I.custom(B=1, Hq=2, Hkv=1, L=600, lo=5, hi=60, k=0, wid=109), 10 ** 6, 2, 0),
    ("unbounded-budget", I.custom(B=2, Hq=4, Hkv=2, L=640, lo=5, hi=60, k=5, wid=105), 10 ** 6, 0, 5),
    ("geometric", I.custom(B=2, Hq=4, Hkv=1, L=3000, lo=1, hi=1024, kind="geometric", mean=40.0, k=6, wid=108),
     400, 2, 40),
]


@needs_gpu
@pytest.mark.parametrize("case", CASES, ids=[c[0] for c in CASES])
def test_budget_small_all_stages(lib, case):
    name, w, budget, recent, k_max = case
    d = I.make_inputs(w)
    t = P.to_dev(d)
    layer = lib.DHSAPrefill(w.B, w.Hq, w.Hkv, w.L, t["off"], t["n_chunks"], k_max, budget=budget, recent=recent)
    O = layer.run(t["Q"], t["K"], t["V"])
    torch.cuda.synchronize()
    assert lib.check_device_status() == 0
    Q, K, V = (ora.bf16_to_f64(d[x]) for x in "QKV")
    off, nc = d["off"], d["n_chunks"]
    nmax = off.shape[1] - 1
    Qp = ora.chunk_pool(Q, off, nc, nmax)
    Kp = ora.chunk_pool(K, off, nc, nmax)
    S = ora.chunk_scores(Qp, Kp, nc)
    sel_gpu = P.gpu_sel_rows(layer.sel, layer.n_sel)
    rows, mism = _compare_budget(S, off, nc, sel_gpu, budget, recent, k_max)
    # padded rows, CSR from the GPU's own selection, attention over it
    n_sel = layer.n_sel.cpu().numpy()
    for b in range(w.B):
        assert np.all(n_sel[b, :, int(nc[b]):] == 0)
    rp, ci, cost = ora.block_csr(sel_gpu, off, nc, nmax)
    assert np.array_equal(layer.row_ptr.cpu().numpy(), rp)
    assert np.array_equal(layer.col_idx.cpu().numpy()[: rp[-1]], ci)
    assert np.array_equal(layer.cost.cpu().numpy(), cost)
    O_ref = ora.attn_sparse(Q, K, V, off, nc, sel_gpu)
    mx, mean = P.compare_out(O, O_ref)
    print(f"{name}: rows={rows} near-tie swaps={mism} max_abs={mx:.3e} mean_abs={mean:.3e}")
    assert mx <= P.MAX_ABS and mean <= P.MEAN_ABS


@needs_gpu
def test_budget_per_row_vector(lib):
    """Query-dependent budgets: an int32 [B, Hq, Nmax] tensor of per-row budgets."""
    w = I.custom(B=2, Hq=4, Hkv=2, L=2000, lo=8, hi=160, k=4, wid=110)
    d = I.make_inputs(w)
    t = P.to_dev(d)
    off, nc = d["off"], d["n_chunks"]
    nmax = off.shape[1] - 1
    rng = np.random.default_rng(5)
    budgets = rng.integers(0, 1200, (w.B, w.Hq, nmax)).astype(np.int32)
    budgets[0, 0, :] = 0
    budgets[1, 1, :] = 10 ** 6
    Qp = lib.chunk_pool(t["Q"], t["off"], t["n_chunks"])
    Kp = lib.chunk_pool(t["K"], t["off"], t["n_chunks"])
    sel, n_sel = lib.chunk_score_select_budget(Qp, Kp, t["off"], t["n_chunks"], torch.from_numpy(budgets).cuda(),
                                               recent=1, k_max=20)
    torch.cuda.synchronize()
    assert lib.check_device_status() == 0
    S = ora.chunk_scores(ora.chunk_pool(ora.bf16_to_f64(d["Q"]), off, nc, nmax),
                         ora.chunk_pool(ora.bf16_to_f64(d["K"]), off, nc, nmax), nc)
    rows, mism = _compare_budget(S, off, nc, P.gpu_sel_rows(sel, n_sel), budgets, 1, 20)
    print(f"per-row budgets: rows={rows} near-tie swaps={mism}")


@needs_gpu
def test_budget_exact_ties_lower_index(lib):
    """All pooled keys equal: every score of a row ties, so the ranked order
    is the chunk index and the kept set is fixed exactly."""
    w = I.custom(B=1, Hq=2, Hkv=1, L=900, lo=10, hi=40, k=3, wid=111)
    d = I.make_inputs(w)
    t = P.to_dev(d)
    Qp = lib.chunk_pool(t["Q"], t["off"], t["n_chunks"])
    Kp = lib.chunk_pool(t["K"], t["off"], t["n_chunks"])
    Kp[:] = Kp[:, :, :1, :].clone()          # one pooled key for every chunk
    sel, n_sel = lib.chunk_score_select_budget(Qp, Kp, t["off"], t["n_chunks"], 100, recent=1, k_max=10)
    torch.cuda.synchronize()
    off, nc = d["off"], d["n_chunks"]
    lens = np.diff(off[0, : int(nc[0]) + 1])
    got = P.gpu_sel_rows(sel, n_sel)
    for h in range(w.Hq):
        for i in range(int(nc[0])):
            want = ora.select_budget_row(np.zeros(int(nc[0])), lens, i, 100, 1, 10)
            assert got[0][h][i].tolist() == want.tolist(), (h, i)


@needs_gpu
def test_budget_full_size_128k_sampled_heads(lib):
    """The 128K layer with a token budget near its top-k density (17 chunks of
    ~160 tokens) and a 2-chunk window: every selection row of two heads
    against the oracle, and sampled outputs."""
    w = I.WORKLOADS["llama8b-128k"]
    d = I.make_inputs(w)
    t = P.to_dev(d)
    budget, recent, k_max = 2720, 2, 48
    layer = lib.DHSAPrefill(w.B, w.Hq, w.Hkv, w.L, t["off"], t["n_chunks"], k_max, budget=budget, recent=recent)
    O = layer.run(t["Q"], t["K"], t["V"])
    torch.cuda.synchronize()
    assert lib.check_device_status() == 0
    off, nc = d["off"], d["n_chunks"]
    nmax = off.shape[1] - 1
    heads = [0, w.Hq - 1]
    sel_gpu = P.gpu_sel_rows(layer.sel, layer.n_sel)
    total = 0
    for hq in heads:
        hkv = hq // w.G
        Qp = ora.chunk_pool(ora.bf16_to_f64(d["Q"][:, hq:hq + 1]), off, nc, nmax)
        Kp = ora.chunk_pool(ora.bf16_to_f64(d["K"][:, hkv:hkv + 1]), off, nc, nmax)
        S = ora.chunk_scores(Qp, Kp, nc)
        _, mism = _compare_budget(S, off, nc, [[sel_gpu[b][hq]] for b in range(w.B)], budget, recent, k_max,
                                  heads=[hq])
        total += mism
    rng = np.random.default_rng(9)
    n = int(nc[0])
    errs = []
    for hq in heads:
        hkv = hq // w.G
        Qf = ora.bf16_to_f64(d["Q"][0, hq]).astype(np.float32)
        Kf = ora.bf16_to_f64(d["K"][0, hkv]).astype(np.float32)
        Vf = ora.bf16_to_f64(d["V"][0, hkv]).astype(np.float32)
        for i in sorted({0, 1, n - 1, *rng.choice(n, 12, replace=False).tolist()}):
            s, e = int(off[0, i]), int(off[0, i + 1])
            ref = ora.attn_chunk(Qf, Kf, Vf, off[0], sel_gpu[0][hq][i], i, P.scale(), np.float32)
            errs.append(np.abs(O[0, hq, s:e].float().cpu().numpy() - ref))
    err = np.concatenate([x.ravel() for x in errs])
    print(f"128K budget: near-tie swaps={total} sampled max_abs={err.max():.3e} mean_abs={err.mean():.3e}")
    assert err.max() <= P.MAX_ABS and err.mean() <= P.MEAN_ABS
