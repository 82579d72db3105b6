"""The routing variants agree bit for bit: the separate launches with the
scan-and-fill CSR build (reference), the selection that writes its CSR rows
directly (the layer's default under the top-k rule), and the one-launch
routing (pooling, key norms, score tiles, selection and CSR in one
cooperative kernel). The layer built on the one-launch routing matches the
CPU oracle."""
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


CASES = {
    "tiny": I.WORKLOADS["tiny"],
    "batch2-gqa8": I.custom(B=2, Hq=8, Hkv=1, L=777, lo=3, hi=90, k=4, wid=103),
    "k0-diag-only": I.custom(B=1, Hq=2, Hkv=1, L=1000, lo=1, hi=300, k=0, wid=104),
    "k-all-dense": I.custom(B=2, Hq=4, Hkv=2, L=640, lo=5, hi=60, k=100000, wid=105),
    "short-seq": I.custom(B=3, Hq=2, Hkv=1, L=37, lo=1, hi=9, k=2, wid=107),
    "geometric": I.custom(B=2, Hq=4, Hkv=1, L=3000, lo=1, hi=1024, kind="geometric", mean=40.0, k=6, wid=108),
    "many-chunks": I.custom(B=1, Hq=2, Hkv=1, L=16000, lo=1, hi=3, k=5, wid=120),
    # ~12000 chunks: one head's packed scores (~288 MB) exceed the 256 MiB
    # score area, so the four heads run as four head batches, with a barrier
    # between a batch's selection and the next batch's score tiles
    # overwriting the same scores (and key norms from the first batch)
    "four-head-batches": I.custom(B=1, Hq=4, Hkv=1, L=24000, lo=1, hi=3, k=5, wid=122),
    # ~7000 chunks, two heads per batch: the second kv group's norms come
    # from the second batch's score tiles
    "two-head-batches": I.custom(B=1, Hq=4, Hkv=2, L=14000, lo=1, hi=3, k=5, wid=123),
    "ragged-64k": I.WORKLOADS["ragged-64k"],
    "llama8b-32k": I.WORKLOADS["llama8b-32k"],
}


def _layers(lib, d, w):
    t = P.to_dev(d)
    a = lib.DHSAPrefill(w.B, w.Hq, w.Hkv, w.L, t["off"], t["n_chunks"], w.k, csr_from_selection=False)
    f = lib.DHSAPrefill(w.B, w.Hq, w.Hkv, w.L, t["off"], t["n_chunks"], w.k, fused_routing=True)
    return t, a, f


@needs_gpu
@pytest.mark.parametrize("name", list(CASES))
def test_routing_variants_agree(lib, name):
    w = CASES[name]
    d = I.make_inputs(w, with_v=False)
    t, a, f = _layers(lib, d, w)
    c = lib.DHSAPrefill(w.B, w.Hq, w.Hkv, w.L, t["off"], t["n_chunks"], w.k)
    for lay in (a, c, f):
        lay.col_idx.fill_(-7)
        lay.routing(t["Q"], t["K"])
    torch.cuda.synchronize()
    assert lib.check_device_status() == 0
    nnz = int(a.row_ptr[-1])
    for other in (c, f):
        for x in ("Qp", "Kp", "sel", "n_sel", "row_ptr", "cost"):
            assert torch.equal(getattr(a, x), getattr(other, x)), x
        assert torch.equal(a.col_idx[:nnz], other.col_idx[:nnz])


@needs_gpu
def test_fused_routing_layer_matches_oracle(lib):
    w = I.custom(B=2, Hq=4, Hkv=2, L=1500, lo=20, hi=300, k=4, wid=121)
    d = I.make_inputs(w)
    t, _, f = _layers(lib, d, w)
    O = f.run(t["Q"], t["K"], t["V"])
    torch.cuda.synchronize()
    assert lib.check_device_status() == 0
    Q, K, V, Qp, Kp, S, sel_ora = P.oracle_full(d, w.k)
    sel_gpu = P.gpu_sel_rows(f.sel, f.n_sel)
    rows, mism = P.compare_selection(S, sel_ora, sel_gpu, d["n_chunks"], w.k)
    O_ref = ora.attn_sparse(Q, K, V, d["off"], d["n_chunks"], sel_gpu)
    mx, mean = P.compare_out(O, O_ref)
    assert mx <= P.MAX_ABS and mean <= P.MEAN_ABS
