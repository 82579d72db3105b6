"""GPU parity: every stage of the CUDA path against the CPU oracle, on the
same seeded inputs, through the C ABI (ctypes binding).

Bars: pooled vectors within 2e-5 relative of the fp64 oracle; selected chunk
sets identical except rows the oracle flags as near-ties (gap below 1e-5 of
the row's largest |score|), which are counted and must still be valid; CSR
bit-exact; attention output max-abs <= 2e-2 and mean-abs <= 2e-3 against the
oracle (bf16 output vs fp64/fp32 oracle).
"""
import math

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


# small workloads that finish in seconds on the oracle; they span several
# 128-row query tiles and 128-slot key tiles and end on ragged tails
SMALL = {
    "tiny": I.WORKLOADS["tiny"],
    "ones-and-twos": I.custom(B=1, Hq=2, Hkv=2, L=301, lo=1, hi=2, k=5, wid=101),
    "long-chunks": I.custom(B=1, Hq=4, Hkv=1, L=1500, lo=100, hi=700, k=2, wid=102),
    "batch2-gqa8": I.custom(B=2, Hq=8, Hkv=1, L=777, lo=3, hi=90, k=4, wid=103),
    "k0-diag-only": I.custom(B=1, Hq=2, Hkv=1, L=1000, lo=1, hi=300, k=0, wid=104),
    "k-all-dense": I.custom(B=2, Hq=4, Hkv=2, L=640, lo=5, hi=60, k=100000, wid=105),
    "single-chunk": I.custom(B=1, Hq=2, Hkv=1, L=200, lo=500, hi=600, k=3, wid=106),
    "short-seq": I.custom(B=3, Hq=2, Hkv=1, L=37, lo=1, hi=9, k=2, wid=107),
    # fewer than four Q rows in all: the attention loads Q through four views
    # of every fourth row, and these leave some views empty
    "three-rows": I.custom(B=1, Hq=1, Hkv=1, L=3, lo=1, hi=2, k=2, wid=116),
    "one-row": I.custom(B=1, Hq=1, Hkv=1, L=1, lo=1, hi=2, k=2, wid=117),
    "geometric": I.custom(B=2, Hq=4, Hkv=1, L=3000, lo=1, hi=1024, kind="geometric", mean=40.0, k=6, wid=108),
}


def _run_gpu(lib, d, k):
    t = P.to_dev(d)
    w = d["workload"]
    layer = lib.DHSAPrefill(w.B, w.Hq, w.Hkv, w.L, t["off"], t["n_chunks"], k)
    O = layer.run(t["Q"], t["K"], t["V"])
    torch.cuda.synchronize()
    assert lib.check_device_status() == 0
    return layer, O


@needs_gpu
@pytest.mark.parametrize("name", list(SMALL))
def test_small_workload_all_stages(lib, name):
    w = SMALL[name]
    d = I.make_inputs(w)
    k = w.k
    layer, O = _run_gpu(lib, d, k)
    Q, K, V, Qp, Kp, S, sel_ora = P.oracle_full(d, k)

    # a1 pooling
    for got, ref in ((layer.Qp, Qp), (layer.Kp, Kp)):
        g = got.cpu().numpy().astype(np.float64)
        assert np.all(np.abs(g - ref) <= P.POOL_RTOL * (np.abs(ref) + 1.0))

    # a2-a3 selection
    sel_gpu = P.gpu_sel_rows(layer.sel, layer.n_sel)
    rows, mism = P.compare_selection(S, sel_ora, sel_gpu, d["n_chunks"], k)
    n_sel = layer.n_sel.cpu().numpy()
    for b in range(w.B):
        n = int(d["n_chunks"][b])
        assert np.all(n_sel[b, :, n:] == 0)
        assert np.all(n_sel[b, :, :n] == np.minimum(k, np.arange(n)) + 1)

    # a4 CSR, from the GPU's own selection
    nmax = d["off"].shape[1] - 1
    rp, ci, cost = ora.block_csr(sel_gpu, d["off"], d["n_chunks"], nmax)
    assert np.array_equal(layer.row_ptr.cpu().numpy(), rp)
    assert np.array_equal(layer.col_idx.cpu().numpy()[: rp[-1]], ci)
    assert np.array_equal(layer.cost.cpu().numpy(), cost)

    # a5 attention over the GPU's selection (identical to the oracle's except
    # accepted near-tie rows)
    O_ref = ora.attn_sparse(Q, K, V, d["off"], d["n_chunks"], sel_gpu)
    mx, mean = P.compare_out(O, O_ref)
    print(f"{name}: rows={rows} near-tie swaps={mism} max_abs={mx:.3e} mean_abs={mean:.3e}")
    assert mx <= P.MAX_ABS and mean <= P.MEAN_ABS


@needs_gpu
def test_k_all_equals_dense(lib):
    w = SMALL["k-all-dense"]
    d = I.make_inputs(w)
    _, O = _run_gpu(lib, d, w.k)
    Q, K, V = (ora.bf16_to_f64(d[x]) for x in "QKV")
    mx, mean = P.compare_out(O, ora.attn_dense(Q, K, V))
    assert mx <= P.MAX_ABS and mean <= P.MEAN_ABS


def _tie_inputs(kind):
    """Equal-length chunks whose pooled keys tie exactly: "pairs" copies the K
    rows of chunk 2c onto chunk 2c+1, "all" gives every key token the same row."""
    w = I.custom(B=1, Hq=4, Hkv=2, L=16 * 90, lo=16, hi=16, k=7, wid=110 if kind == "pairs" else 111)
    d = I.make_inputs(w)
    K = d["K"]
    if kind == "pairs":
        for c in range(0, 89, 2):
            K[:, :, 16 * (c + 1):16 * (c + 2)] = K[:, :, 16 * c:16 * (c + 1)]
    else:
        K[:] = K[:, :, :1]
    return w, d


@needs_gpu
@pytest.mark.parametrize("kind", ["pairs", "all"])
def test_exact_ties_resolve_to_lower_index(lib, kind):
    """Exactly tied chunk scores (the degenerate case of the ranking) must be
    resolved like the oracle: the lower chunk index wins, with no tolerance."""
    w, d = _tie_inputs(kind)
    layer, O = _run_gpu(lib, d, w.k)
    Q, K, V, Qp, Kp, S, sel_ora = P.oracle_full(d, w.k)
    sel_gpu = P.gpu_sel_rows(layer.sel, layer.n_sel)
    for h in range(w.Hq):
        for i in range(int(d["n_chunks"][0])):
            assert np.array_equal(sel_gpu[0][h][i], sel_ora[0][h][i]), (kind, h, i)
    if kind == "all":
        for h in range(w.Hq):
            for i in range(int(d["n_chunks"][0])):
                assert list(sel_gpu[0][h][i]) == list(range(min(w.k, i))) + [i]
    mx, mean = P.compare_out(O, ora.attn_sparse(Q, K, V, d["off"], d["n_chunks"], sel_gpu))
    assert mx <= P.MAX_ABS and mean <= P.MEAN_ABS


@needs_gpu
def test_many_chunks_head_batched_scores(lib):
    """~8000 one- or two-token chunks per sequence: the score workspace no
    longer holds every head at once, so the score/top-k call loops over head
    batches. Selection is checked row by row against the oracle."""
    w = I.custom(B=1, Hq=4, Hkv=2, L=12000, lo=1, hi=2, k=12, wid=112)
    d = I.make_inputs(w)
    nmax = d["off"].shape[1] - 1
    assert 4 * nmax * (nmax - 1) // 2 * w.B * w.Hq > (256 << 20)
    layer, O = _run_gpu(lib, d, w.k)
    Q, K, V = (ora.bf16_to_f64(d[x]) for x in "QKV")
    Qp = ora.chunk_pool(Q, d["off"], d["n_chunks"], nmax)
    Kp = ora.chunk_pool(K, d["off"], d["n_chunks"], nmax)
    S = ora.chunk_scores(Qp, Kp, d["n_chunks"])
    sel_ora = ora.select(S, d["n_chunks"], w.k)
    sel_gpu = P.gpu_sel_rows(layer.sel, layer.n_sel)
    rows, mism = P.compare_selection(S, sel_ora, sel_gpu, d["n_chunks"], w.k)
    print(f"many-chunks: rows={rows} near-tie swaps={mism}")
    rng = np.random.default_rng(3)
    n = int(d["n_chunks"][0])
    for i in rng.choice(n, size=40, replace=False):
        s0, e0 = int(d["off"][0, i]), int(d["off"][0, i + 1])
        for h in (0, 3):
            ref = ora.attn_chunk(Q[0, h], K[0, h // 2], V[0, h // 2], d["off"][0], sel_gpu[0][h][i], int(i), P.scale())
            assert np.abs(O[0, h, s0:e0].float().cpu().numpy() - ref).max() <= P.MAX_ABS


@needs_gpu
def test_two_calls_same_result(lib):
    d = I.make_inputs(SMALL["geometric"])
    t = P.to_dev(d)
    w = d["workload"]
    layer = lib.DHSAPrefill(w.B, w.Hq, w.Hkv, w.L, t["off"], t["n_chunks"], w.k)
    O1 = layer.run(t["Q"], t["K"], t["V"]).clone()
    O2 = layer.run(t["Q"], t["K"], t["V"])
    torch.cuda.synchronize()
    assert torch.equal(O1, O2)


def _sample_chunks(n, lens, rng, extra=()):
    pick = {0, n - 1, int(np.argmax(lens))}
    pick.update(int(x) for x in rng.choice(n, size=min(n, 24), replace=False))
    pick.update(int(x) for x in extra)
    return sorted(pick)


@needs_gpu
@pytest.mark.parametrize("name", ["qwen3b-8k", "llama8b-32k", "llama8b-128k", "ragged-64k"])
def test_full_size_sampled(lib, name):
    """Full-size workloads in the benchmark's launch configuration; the
    oracle checks every pooled vector and selection row of two sampled heads
    and the outputs of sampled query chunks."""
    w = I.WORKLOADS[name]
    d = I.make_inputs(w)
    layer, O = _run_gpu(lib, d, w.k)
    off, nc = d["off"], d["n_chunks"]
    nmax = off.shape[1] - 1
    rng = np.random.default_rng(7)
    heads = sorted({0, w.Hq - 1})
    sel_gpu = P.gpu_sel_rows(layer.sel, layer.n_sel)
    Qp_g, Kp_g = layer.Qp.cpu().numpy(), layer.Kp.cpu().numpy()
    total_mism = 0
    for hq in heads:
        hkv = hq // w.G
        Qp = ora.chunk_pool(ora.bf16_to_f64(d["Q"][:, hq:hq + 1]), off, nc, nmax)
        Kp = ora.chunk_pool(ora.bf16_to_f64(d["K"][:, hkv:hkv + 1]), off, nc, nmax)
        assert np.all(np.abs(Qp_g[:, hq:hq + 1] - Qp) <= P.POOL_RTOL * (np.abs(Qp) + 1.0))
        assert np.all(np.abs(Kp_g[:, hkv:hkv + 1] - Kp) <= P.POOL_RTOL * (np.abs(Kp) + 1.0))
        S = ora.chunk_scores(Qp, Kp, nc)
        sel_o = ora.select(S, nc, w.k)
        _, mism = P.compare_selection(S, sel_o, [[sel_gpu[b][hq]] for b in range(w.B)], nc, w.k)
        total_mism += mism
    # needles: every planted pair is selected by the GPU
    for b in range(w.B):
        for (hq, i, j) in d["needles"][b]:
            assert j in sel_gpu[b][hq][i]
    # sampled outputs over the GPU selection, fp32 oracle attention
    Qf = ora.bf16_to_f64(d["Q"][:, heads]).astype(np.float32)
    errs = []
    for b in range(w.B):
        n = int(nc[b])
        lens = np.diff(off[b, : n + 1])
        for hi, hq in enumerate(heads):
            hkv = hq // w.G
            Kf = ora.bf16_to_f64(d["K"][b, hkv]).astype(np.float32)
            Vf = ora.bf16_to_f64(d["V"][b, hkv]).astype(np.float32)
            needle_rows = [i for (h, i, _) in d["needles"][b] if h == hq][:4]
            for i in _sample_chunks(n, lens, rng, needle_rows):
                s, e = int(off[b, i]), int(off[b, i + 1])
                ref = ora.attn_chunk(Qf[b, hi], Kf, Vf, off[b], sel_gpu[b][hq][i], i, P.scale(), np.float32)
                got = O[b, hq, s:e].float().cpu().numpy()
                errs.append(np.abs(got - ref))
    err = np.concatenate([e.ravel() for e in errs])
    print(f"{name}: near-tie swaps={total_mism} sampled max_abs={err.max():.3e} mean_abs={err.mean():.3e}")
    assert err.max() <= P.MAX_ABS and err.mean() <= P.MEAN_ABS


@needs_gpu
def test_ragged_k_all_sampled_vs_dense(lib):
    """The ragged 64K workload with k = all causal chunks equals dense causal
    attention (sampled query chunks of two heads, checked against the
    oracle's textbook dense attention on the tokens up to each chunk)."""
    w = I.WORKLOADS["ragged-64k"]
    d = I.make_inputs(w)
    _, O = _run_gpu(lib, d, 1 << 20)
    off, nc = d["off"], d["n_chunks"]
    rng = np.random.default_rng(11)
    errs = []
    for b in range(w.B):
        n = int(nc[b])
        for hq in (1, w.Hq - 2):
            hkv = hq // w.G
            for i in sorted(rng.choice(n, size=6, replace=False)):
                s, e = int(off[b, i]), int(off[b, i + 1])
                q = ora.bf16_to_f64(d["Q"][b, hq, s:e]).astype(np.float32)
                kk = ora.bf16_to_f64(d["K"][b, hkv, :e]).astype(np.float32)
                v = ora.bf16_to_f64(d["V"][b, hkv, :e]).astype(np.float32)
                logits = (q @ kk.T) * np.float32(P.scale())
                logits = np.where(np.arange(e)[None, :] <= np.arange(s, e)[:, None], logits, -np.inf)
                p = np.exp(logits - logits.max(1, keepdims=True))
                ref = (p @ v) / p.sum(1, keepdims=True)
                errs.append(np.abs(O[b, hq, s:e].float().cpu().numpy() - ref).ravel())
    err = np.concatenate(errs)
    assert err.max() <= P.MAX_ABS and err.mean() <= P.MEAN_ABS


@needs_gpu
def test_validate_offsets_flags_bad_table(lib):
    off = torch.tensor([[0, 5, 5, 9]], dtype=torch.int32, device="cuda")   # not strictly increasing
    nc = torch.tensor([3], dtype=torch.int32, device="cuda")
    lib.check_device_status()
    lib.validate_offsets(off, nc, 9)
    with pytest.raises(lib.DHSAError) as e:
        lib.check_device_status()
    assert e.value.flags & lib.DEVFLAG_BAD_OFFSETS
    good = torch.tensor([[0, 5, 7, 9]], dtype=torch.int32, device="cuda")
    lib.validate_offsets(good, nc, 9)
    assert lib.check_device_status() == 0


@needs_gpu
def test_pool_qk_matches_separate_pools(lib):
    """The one-launch pooling of Q and K is bit-identical to two dhsa_chunk_pool calls."""
    w = I.custom(B=2, Hq=8, Hkv=2, L=3000, lo=1, hi=400, kind="geometric", mean=50.0, k=4, wid=112)
    d = I.make_inputs(w)
    t = P.to_dev(d)
    Qp, Kp = lib.chunk_pool_qk(t["Q"], t["K"], t["off"], t["n_chunks"])
    Qs = lib.chunk_pool(t["Q"], t["off"], t["n_chunks"])
    Ks = lib.chunk_pool(t["K"], t["off"], t["n_chunks"])
    torch.cuda.synchronize()
    assert torch.equal(Qp, Qs) and torch.equal(Kp, Ks)


@needs_gpu
def test_host_streamed_layers_match_direct_runs(lib):
    """Three layers submitted back to back from pinned host memory (copies of
    neighbouring layers overlapping the compute) give exactly the outputs of
    direct runs on device-resident inputs."""
    w = I.custom(B=1, Hq=8, Hkv=2, L=4000, lo=10, hi=300, k=4, wid=113)
    d = I.make_inputs(w)
    t = P.to_dev(d)
    layer = lib.DHSAPrefill(w.B, w.Hq, w.Hkv, w.L, t["off"], t["n_chunks"], w.k)
    rng = np.random.default_rng(21)
    hosts, refs = [], []
    for s in range(3):
        perm = rng.permutation(w.L)
        hq = {x: torch.from_numpy(np.ascontiguousarray(d[x][:, :, perm])).view(torch.bfloat16).pin_memory()
              for x in "QKV"}
        hosts.append(hq)
        refs.append(layer.run(*(hq[x].cuda() for x in "QKV")).clone())
    torch.cuda.synchronize()
    runner = lib.HostStreamedPrefill(layer)
    outs = [torch.empty(hosts[0]["Q"].shape, dtype=torch.bfloat16).pin_memory() for _ in range(3)]
    for hq, oh in zip(hosts, outs):
        runner.submit(hq["Q"], hq["K"], hq["V"], oh)
    runner.synchronize()
    assert lib.check_device_status() == 0
    for oh, ref in zip(outs, refs):
        assert torch.equal(oh, ref.cpu())


@needs_gpu
def test_graphed_layer_matches_eager(lib):
    """A layer captured as a CUDA graph and replayed over refilled inputs gives
    exactly the eager outputs."""
    w = I.custom(B=2, Hq=8, Hkv=2, L=2500, lo=5, hi=200, kind="geometric", mean=60.0, k=5, wid=114)
    d = I.make_inputs(w)
    t = P.to_dev(d)
    layer = lib.DHSAPrefill(w.B, w.Hq, w.Hkv, w.L, t["off"], t["n_chunks"], w.k)
    Q, K, V = (t[x].clone() for x in "QKV")
    g = lib.GraphedPrefill(layer, Q, K, V)
    rng = np.random.default_rng(4)
    for s in range(3):
        perm = torch.from_numpy(rng.permutation(w.L)).cuda()
        newQ, newK, newV = (t[x][:, :, perm].contiguous() for x in "QKV")
        Q.copy_(newQ), K.copy_(newK), V.copy_(newV)
        out = g.replay().clone()
        ref_layer = lib.DHSAPrefill(w.B, w.Hq, w.Hkv, w.L, t["off"], t["n_chunks"], w.k)
        ref = ref_layer.run(newQ, newK, newV)
        torch.cuda.synchronize()
        assert lib.check_device_status() == 0
        assert torch.equal(out, ref)
