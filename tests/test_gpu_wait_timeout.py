"""Failure detection without a device fault.

Every wait of the pipelined kernels is bounded: once it has waited longer
than its limit it records DHSA_DEVFLAG_WAIT_TIMEOUT and the kernel unwinds
instead of hanging. The library's test hook (include/dhsa.h, 5) makes such a
wait run out on purpose -- the attention kernel's scheduler publishes no
work item, so the first wait of every other role, which comes before any
copy or MMA, runs out; in the fused routing, block 0 reaches the first grid
barrier late. Nothing traps and no access leaves its buffer. The tests check
that the call returns, that the flag is reported, and that the next normal
call in the same process is clean and correct.

Inconsistent offsets tables are handled the same way: pooling clamps them
(no read leaves the head's rows) and the attention's work-list builder skips
the batch element; both report DHSA_DEVFLAG_BAD_OFFSETS.
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


def _flags(lib):
    try:
        return lib.check_device_status()
    except lib.DHSAError as e:
        return e.flags


def _layer(lib, w):
    d = I.make_inputs(w)
    t = P.to_dev(d)
    layer = lib.DHSAPrefill(w.B, w.Hq, w.Hkv, w.L, t["off"], t["n_chunks"], w.k)
    return d, t, layer


@needs_gpu
def test_attention_wait_runs_out_then_recovers(lib):
    w = I.custom(B=1, Hq=4, Hkv=2, L=1200, lo=10, hi=200, k=3, wid=140)
    d, t, layer = _layer(lib, w)
    layer.routing(t["Q"], t["K"])
    torch.cuda.synchronize()
    assert _flags(lib) == 0
    O = torch.full_like(t["Q"], 7.0)

    def attend():
        lib.sparse_attn_fwd(t["Q"], t["K"], t["V"], t["off"], t["n_chunks"], layer.row_ptr, layer.col_idx, out=O)

    lib.debug_arm_wait_timeout(1, 50_000)            # 50 us
    attend()
    flags = _flags(lib)
    assert flags & lib.DEVFLAG_WAIT_TIMEOUT, flags
    # nothing was written: the kernel left before any item
    assert torch.all(O.float() == 7.0)
    # the hook is one-shot: the next call runs normally and matches the oracle
    attend()
    assert _flags(lib) == 0
    Q, K, V, Qp, Kp, S, sel = P.oracle_full(d, w.k)
    ref = ora.attn_sparse(Q, K, V, d["off"], d["n_chunks"], P.gpu_sel_rows(layer.sel, layer.n_sel))
    mx, mean = P.compare_out(O, ref)
    assert mx <= P.MAX_ABS and mean <= P.MEAN_ABS


@needs_gpu
def test_fused_routing_barrier_runs_out_then_recovers(lib):
    w = I.custom(B=2, Hq=4, Hkv=1, L=3000, lo=5, hi=120, k=4, wid=141)
    d = I.make_inputs(w, with_v=False)
    t = P.to_dev(d)
    a = lib.DHSAPrefill(w.B, w.Hq, w.Hkv, w.L, t["off"], t["n_chunks"], w.k)
    f = lib.DHSAPrefill(w.B, w.Hq, w.Hkv, w.L, t["off"], t["n_chunks"], w.k, fused_routing=True)
    a.routing(t["Q"], t["K"])
    torch.cuda.synchronize()
    assert _flags(lib) == 0
    lib.debug_arm_wait_timeout(2, 50_000)
    f.routing(t["Q"], t["K"])
    flags = _flags(lib)
    assert flags & lib.DEVFLAG_WAIT_TIMEOUT, flags
    f.routing(t["Q"], t["K"])
    assert _flags(lib) == 0
    for x in ("Qp", "Kp", "sel", "n_sel", "row_ptr"):
        assert torch.equal(getattr(a, x), getattr(f, x)), x


@needs_gpu
def test_disarmed_hook_changes_nothing(lib):
    w = I.custom(B=1, Hq=2, Hkv=1, L=500, lo=10, hi=90, k=2, wid=142)
    d, t, layer = _layer(lib, w)
    lib.debug_arm_wait_timeout(1, 50_000)
    lib.debug_arm_wait_timeout(0)
    O = layer.run(t["Q"], t["K"], t["V"])
    assert _flags(lib) == 0
    Q, K, V, Qp, Kp, S, sel = P.oracle_full(d, w.k)
    ref = ora.attn_sparse(Q, K, V, d["off"], d["n_chunks"], P.gpu_sel_rows(layer.sel, layer.n_sel))
    mx, mean = P.compare_out(O, ref)
    assert mx <= P.MAX_ABS and mean <= P.MEAN_ABS


@needs_gpu
def test_pooling_clamps_bad_offsets(lib):
    w = I.custom(B=2, Hq=2, Hkv=1, L=300, lo=10, hi=60, k=2, wid=143)
    d = I.make_inputs(w, with_v=False)
    t = P.to_dev(d)
    good = lib.chunk_pool(t["K"], t["off"], t["n_chunks"])
    torch.cuda.synchronize()
    assert _flags(lib) == 0
    off = d["off"].copy()
    n1 = int(d["n_chunks"][1])
    off[1, n1 - 1] = 5 * w.L          # a bound far past L in batch element 1
    bad = lib.chunk_pool(t["K"], torch.from_numpy(off).cuda(), t["n_chunks"])
    assert _flags(lib) & lib.DEVFLAG_BAD_OFFSETS
    # batch element 0 is untouched by the bad row of element 1
    assert torch.equal(good[0], bad[0])
    assert torch.isfinite(bad).all()
    nc = d["n_chunks"].copy()
    nc[0] = 10 ** 6                    # a chunk count past Nmax
    lib.chunk_pool(t["K"], t["off"], torch.from_numpy(nc).cuda())
    assert _flags(lib) & lib.DEVFLAG_BAD_OFFSETS
    lib.chunk_pool(t["K"], t["off"], t["n_chunks"])
    assert _flags(lib) == 0


@needs_gpu
def test_attention_skips_batch_with_bad_offsets(lib):
    w = I.custom(B=2, Hq=2, Hkv=1, L=400, lo=10, hi=60, k=2, wid=144)
    d, t, layer = _layer(lib, w)
    O_good = layer.run(t["Q"], t["K"], t["V"]).clone()
    assert _flags(lib) == 0
    off = d["off"].copy()
    off[1, 0] = 3                      # element 1's table must start at 0
    off_bad = torch.from_numpy(off).cuda()
    O = torch.full_like(t["Q"], 5.0)
    lib.sparse_attn_fwd(t["Q"], t["K"], t["V"], off_bad, t["n_chunks"], layer.row_ptr, layer.col_idx, out=O)
    assert _flags(lib) & lib.DEVFLAG_BAD_OFFSETS
    assert torch.equal(O[0], O_good[0])           # element 0 computed as before
    assert torch.all(O[1].float() == 5.0)         # element 1 skipped, not written
