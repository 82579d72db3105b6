"""GPU parity of the short-tile attention kernel (query tiles of at most 64
rows, keys on the MMA's M side) against the CPU oracle, under both tile
policies that use it: chunk tails of at most 64 rows (short_tiles=1, next to
128-row tiles of the long-tile kernel) and 64-row tiles only (short_tiles=2).

The layouts put many such tails next to 128-row tiles, one-token chunks and
chunks that straddle key tiles, and one case makes the running column
maximum rise by far more than its headroom after the first key tile. Bars as
in test_gpu_parity.py.
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


def _run(lib, d, k, short_tiles):
    t = P.to_dev(d)
    B, Hq, L = d["Q"].shape[:3]
    Hkv = d["K"].shape[1]
    layer = lib.DHSAPrefill(B, Hq, Hkv, L, t["off"], t["n_chunks"], k, short_tiles=short_tiles)
    O = layer.run(t["Q"], t["K"], t["V"])
    torch.cuda.synchronize()
    assert lib.check_device_status() == 0
    return layer, O


def _check(lib, d, k, short_tiles):
    layer, O = _run(lib, d, k, short_tiles)
    Q, K, V = (ora.bf16_to_f64(d[x]) for x in "QKV")
    sel_gpu = P.gpu_sel_rows(layer.sel, layer.n_sel)
    O_ref = ora.attn_sparse(Q, K, V, d["off"], d["n_chunks"], sel_gpu)
    mx, mean = P.compare_out(O, O_ref)
    print(f"max_abs={mx:.3e} mean_abs={mean:.3e}")
    assert mx <= P.MAX_ABS and mean <= P.MEAN_ABS
    return O


# tails of 1..64 rows after 0, 1 or 2 full tiles, tails just above 64,
# one-token chunks, and a chunk longer than a key tile
EDGE_LENGTHS = [1, 7, 8, 9, 63, 64, 65, 127, 128, 129, 191, 192, 193, 255, 256, 300,
                1, 1, 2, 3, 64, 33, 17, 200, 5]


POLICIES = [1, 2]


@needs_gpu
@pytest.mark.parametrize("short_tiles", POLICIES)
@pytest.mark.parametrize("k", [0, 3, 100000])
def test_edge_lengths(lib, k, short_tiles):
    L = sum(EDGE_LENGTHS)
    w = I.custom(B=1, Hq=4, Hkv=2, L=L, lo=1, hi=64, k=max(k, 1), wid=140)
    d = I.with_lengths(I.make_inputs(w), [EDGE_LENGTHS])
    _check(lib, d, k, short_tiles)


@needs_gpu
@pytest.mark.parametrize("short_tiles", POLICIES)
def test_batch_of_short_chunks(lib, short_tiles):
    # every chunk at most 64 tokens: nearly all work goes to the short-tile kernel
    w = I.custom(B=2, Hq=8, Hkv=2, L=2100, lo=1, hi=64, k=12, wid=141)
    _check(lib, I.make_inputs(w), w.k, short_tiles)


@needs_gpu
@pytest.mark.parametrize("short_tiles", POLICIES)
def test_policies_agree_with_long_tiles(lib, short_tiles):
    # the same layer under policy 0 and under the short-tile policy: equal up
    # to fp32 summation order (a few bf16 ulps)
    w = I.custom(B=2, Hq=4, Hkv=1, L=3000, lo=1, hi=400, kind="geometric", mean=60.0, k=6, wid=143)
    d = I.make_inputs(w)
    _, O0 = _run(lib, d, w.k, 0)
    O0 = O0.clone()
    _, O1 = _run(lib, d, w.k, short_tiles)
    diff = (O0.float() - O1.float()).abs()
    assert diff.max().item() <= 1e-2 and diff.mean().item() <= 1e-4


@needs_gpu
@pytest.mark.parametrize("short_tiles", POLICIES)
def test_column_max_rises_after_first_tile(lib, short_tiles):
    # keys of chunk j scaled by 1 + 3 j: every query's largest logit grows
    # across the key tiles by far more than 2^32 in the softmax's log2 units,
    # so the running maxima rise (and O^T is rescaled) mid-row
    lengths = [[40, 90, 30, 64, 50, 128, 20, 60, 150, 33, 80, 47, 9]]
    L = sum(lengths[0])
    w = I.custom(B=1, Hq=2, Hkv=1, L=L, lo=1, hi=64, k=100000, wid=142)
    d = I.with_lengths(I.make_inputs(w), lengths)
    K = I.bf16_bits_to_f32(d["K"]).copy()
    off = d["off"][0]
    for j in range(int(d["n_chunks"][0])):
        K[:, :, off[j]:off[j + 1]] *= np.float32(1.0 + 3.0 * j)
    d["K"] = I.f32_to_bf16_bits(K)
    layer, O = _run(lib, d, 100000, short_tiles)
    Q, Kf, V = (ora.bf16_to_f64(d[x]) for x in "QKV")
    # the premise: the largest logit of some query grows by > 32 / log2(e)
    s = (Q[0, 0] @ Kf[0, 0].T) * P.scale()
    first = s[-1, : off[1]].max()
    assert s[-1].max() - first > 32 / np.log2(np.e)
    mx, mean = P.compare_out(O, ora.attn_dense(Q, Kf, V))
    print(f"max_abs={mx:.3e} mean_abs={mean:.3e}")
    assert mx <= P.MAX_ABS and mean <= P.MEAN_ABS


@needs_gpu
def test_full_size_128k_tails_on_short_kernel(lib):
    # the 128K layer in the benchmark's configuration with chunk tails of at
    # most 64 rows on the short-tile kernel: sampled chunks (a third of them
    # with such tails) against the fp32 oracle over the GPU's selection, and
    # the whole output against the 128-row policy
    w = I.WORKLOADS["llama8b-128k"]
    d = I.make_inputs(w)
    layer0, O0 = _run(lib, d, w.k, 0)
    O0 = O0.clone()
    layer, O = _run(lib, d, w.k, 1)
    diff = (O0.float() - O.float()).abs()
    assert diff.max().item() <= 1e-2 and diff.mean().item() <= 1e-4
    off, nc = d["off"], d["n_chunks"]
    sel_gpu = P.gpu_sel_rows(layer.sel, layer.n_sel)
    n = int(nc[0])
    lens = np.diff(off[0, : n + 1])
    tails = np.where((lens % 128 != 0) & (lens % 128 <= 64))[0]
    rng = np.random.default_rng(11)
    pick = sorted(set(rng.choice(tails, size=8, replace=False).tolist()) | set(rng.choice(n, size=16, replace=False).tolist()))
    errs = []
    for hq in (0, w.Hq - 1):
        hkv = hq // w.G
        Qf = ora.bf16_to_f64(d["Q"][0, hq]).astype(np.float32)
        Kf = ora.bf16_to_f64(d["K"][0, hkv]).astype(np.float32)
        Vf = ora.bf16_to_f64(d["V"][0, hkv]).astype(np.float32)
        for i in pick:
            s, e = int(off[0, i]), int(off[0, i + 1])
            ref = ora.attn_chunk(Qf, Kf, Vf, off[0], sel_gpu[0][hq][i], i, P.scale(), np.float32)
            errs.append(np.abs(O[0, hq, s:e].float().cpu().numpy() - ref).ravel())
    err = np.concatenate(errs)
    print(f"128K tails on the short kernel: max_abs={err.max():.3e} mean_abs={err.mean():.3e}")
    assert err.max() <= P.MAX_ABS and err.mean() <= P.MEAN_ABS
