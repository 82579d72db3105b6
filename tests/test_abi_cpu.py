"""The C-ABI library builds, loads and exports every function include/dhsa.h
declares; host-side argument checks answer without touching a GPU."""
import ctypes

import pytest

from long_context_prefill_dhsa_b200 import binding, build


@pytest.fixture(scope="module")
def lib():
    build.build()
    return binding.load()


def test_exports_every_declared_function(lib):
    names = binding.header_functions()
    assert len(names) >= 13
    missing = [n for n in names if not hasattr(lib, n)]
    assert not missing, missing
    assert set(names) >= set(binding._SIGNATURES)


def test_status_strings_and_version(lib):
    assert lib.dhsa_version() >= 100
    for code, name in binding.STATUS_NAMES.items():
        assert lib.dhsa_status_string(code).decode() == name
    assert lib.dhsa_status_string(99).decode() == "DHSA_ERR_UNKNOWN"


def test_size_queries(lib):
    assert lib.dhsa_sel_stride(8, 55) == 9
    assert lib.dhsa_sel_stride(100, 55) == 55        # k >= Nmax - 1: every earlier chunk
    assert lib.dhsa_sel_stride(-1, 55) == 0
    assert lib.dhsa_csr_nnz_upper(2, 4, 10, 3) == 2 * 4 * 10 * 4
    # key norms + packed lower-triangle fp32 scores of all heads (they fit in 256 MiB)
    assert lib.dhsa_score_topk_workspace_size(1, 32, 823) >= 4 * 32 * (823 * 822 // 2 + 823)
    # very many chunks: one head's scores at a time (the call loops over heads)
    one_head = 4 * (20000 * 19999 // 2)
    assert one_head <= lib.dhsa_score_topk_workspace_size(1, 32, 20000) < one_head + (4 << 20)
    assert lib.dhsa_sparse_attn_workspace_size(1, 32, 131072, 823) >= 16 * 32 * (823 + 1024)


FAKE = 1 << 20   # a non-null, 16-byte aligned stand-in pointer; never dereferenced


def test_invalid_arguments_rejected_on_host(lib):
    INV, UNS, WS = 1, 2, 5
    # pool: null input, bad sizes, head_dim != 128
    assert lib.dhsa_chunk_pool(None, 1, 1, 8, 128, FAKE, FAKE, 1, FAKE, None) == INV
    assert lib.dhsa_chunk_pool(FAKE, 0, 1, 8, 128, FAKE, FAKE, 1, FAKE, None) == INV
    assert lib.dhsa_chunk_pool(FAKE, 1, 1, 8, 128, FAKE, FAKE, 9, FAKE, None) == INV   # Nmax > L
    assert lib.dhsa_chunk_pool(FAKE + 4, 1, 1, 8, 128, FAKE, FAKE, 1, FAKE, None) == INV  # misaligned
    assert lib.dhsa_chunk_pool(FAKE, 1, 1, 8, 64, FAKE, FAKE, 1, FAKE, None) == UNS
    # score/top-k: k < 0, Hq % Hkv != 0, missing workspace for a large Nmax
    assert lib.dhsa_chunk_score_topk(FAKE, FAKE, 1, 4, 2, 8, FAKE, -1, FAKE, FAKE, None, 0, None) == INV
    assert lib.dhsa_chunk_score_topk(FAKE, FAKE, 1, 3, 2, 8, FAKE, 1, FAKE, FAKE, None, 0, None) == INV
    assert lib.dhsa_chunk_score_topk(FAKE, FAKE, 1, 4, 2, 8, FAKE, 1, FAKE, FAKE, None, 0, None) == WS
    assert lib.dhsa_chunk_score_topk(FAKE, FAKE, 1, 4, 2, 8, FAKE, 1, FAKE, FAKE, FAKE, 64, None) == WS
    # CSR: null output
    assert lib.dhsa_build_block_csr(FAKE, FAKE, 1, 1, 4, 1, FAKE, FAKE, None, FAKE, None, None) == INV
    # attention: head_dim, scale, workspace
    args = [FAKE, FAKE, FAKE, 1, 2, 1, 256, 128, FAKE, FAKE, 4, FAKE, FAKE, None]
    big = lib.dhsa_sparse_attn_workspace_size(1, 2, 256, 4)
    assert lib.dhsa_sparse_attn_fwd(*args, ctypes.c_float(0.1), FAKE, FAKE, big - 16, None) == WS
    assert lib.dhsa_sparse_attn_fwd(*args, ctypes.c_float(-1.0), FAKE, FAKE, big, None) == INV
    args[7] = 96
    assert lib.dhsa_sparse_attn_fwd(*args, ctypes.c_float(0.1), FAKE, FAKE, big, None) == UNS
    args[7] = 128
    args[5] = 3      # Hq % Hkv != 0
    assert lib.dhsa_sparse_attn_fwd(*args, ctypes.c_float(0.1), FAKE, FAKE, big, None) == INV


def test_budget_selection_arguments_rejected_on_host(lib):
    INV, UNS, WS = 1, 2, 5
    cap = lib.dhsa_budget_max_chunks()
    assert cap >= 64
    f = lib.dhsa_chunk_score_select_budget
    #      Qp    Kp    B  Hq Hkv Nmax off   n_ch  budget budgets recent k_max sel   n_sel ws  bytes stream
    assert f(FAKE, FAKE, 1, 4, 2, 8, FAKE, FAKE, 100, None, 0, cap + 1, FAKE, FAKE, FAKE, 1 << 30, None) == UNS
    assert f(FAKE, FAKE, 1, 4, 2, 8, FAKE, FAKE, -1, None, 0, 4, FAKE, FAKE, FAKE, 1 << 30, None) == INV
    assert f(FAKE, FAKE, 1, 4, 2, 8, FAKE, FAKE, 100, None, -1, 4, FAKE, FAKE, FAKE, 1 << 30, None) == INV
    assert f(FAKE, FAKE, 1, 4, 2, 8, FAKE, FAKE, 100, None, 0, -1, FAKE, FAKE, FAKE, 1 << 30, None) == INV
    assert f(FAKE, FAKE, 1, 4, 2, 8, None, FAKE, 100, None, 0, 4, FAKE, FAKE, FAKE, 1 << 30, None) == INV
    assert f(FAKE, FAKE, 1, 3, 2, 8, FAKE, FAKE, 100, None, 0, 4, FAKE, FAKE, FAKE, 1 << 30, None) == INV
    assert f(FAKE, FAKE, 1, 4, 2, 8, FAKE, FAKE, 100, None, 0, 4, FAKE, FAKE, None, 0, None) == WS


def test_tile_policy_arguments_rejected_on_host(lib):
    INV, WS = 1, 5
    ws = lib.dhsa_sparse_attn_tiles_workspace_size
    B, Hq, L, nmax = 1, 32, 131072, 823
    # policy 0 is the plain entry; policy 1 adds one short tile per (b, hq, chunk),
    # policy 2 has 64-row tiles only
    assert ws(B, Hq, L, nmax, 0) == lib.dhsa_sparse_attn_workspace_size(B, Hq, L, nmax)
    assert ws(B, Hq, L, nmax, 1) == ws(B, Hq, L, nmax, 0) + 16 * B * Hq * nmax
    assert ws(B, Hq, L, nmax, 2) == 256 + 16 * B * Hq * (nmax + L // 64)
    assert ws(B, Hq, L, nmax, 3) == 0 and ws(B, Hq, L, nmax, -1) == 0
    f = lib.dhsa_sparse_attn_fwd_tiles
    args = [FAKE, FAKE, FAKE, 1, 2, 1, 256, 128, FAKE, FAKE, 4, FAKE, FAKE, ctypes.c_float(0.1)]
    big = ws(1, 2, 256, 4, 2)
    assert f(*args, 3, FAKE, FAKE, big, None) == INV
    assert f(*args, -1, FAKE, FAKE, big, None) == INV
    assert f(*args, 2, FAKE, FAKE, ws(1, 2, 256, 4, 2) - 16, None) == WS
    assert f(*args, 1, FAKE, None, big, None) == WS


def test_fused_routing_arguments_rejected_on_host(lib):
    INV, UNS, WS = 1, 2, 5
    f = lib.dhsa_route_fused
    ws = lib.dhsa_route_fused_workspace_size(1, 4, 8)
    assert ws == lib.dhsa_score_topk_workspace_size(1, 4, 8) and ws >= 256
    #          Q     K     B  Hq Hkv  L  hd  off   n_ch Nmax k  Qp    Kp    sel   n_sel ws    bytes stream
    assert f(FAKE, FAKE, 1, 4, 2, 64, 128, FAKE, FAKE, 8, -1, FAKE, FAKE, FAKE, FAKE, FAKE, ws, None) == INV
    assert f(FAKE, FAKE, 1, 3, 2, 64, 128, FAKE, FAKE, 8, 2, FAKE, FAKE, FAKE, FAKE, FAKE, ws, None) == INV
    assert f(None, FAKE, 1, 4, 2, 64, 128, FAKE, FAKE, 8, 2, FAKE, FAKE, FAKE, FAKE, FAKE, ws, None) == INV
    assert f(FAKE, FAKE, 1, 4, 2, 64, 128, FAKE, FAKE, 8, 2, FAKE, FAKE, None, FAKE, FAKE, ws, None) == INV
    assert f(FAKE, FAKE, 1, 4, 2, 64, 96, FAKE, FAKE, 8, 2, FAKE, FAKE, FAKE, FAKE, FAKE, ws, None) == UNS
    assert f(FAKE, FAKE, 1, 4, 2, 64, 128, FAKE, FAKE, 8, 2, FAKE, FAKE, FAKE, FAKE, None, ws, None) == WS
    assert f(FAKE, FAKE, 1, 4, 2, 64, 128, FAKE, FAKE, 8, 2, FAKE, FAKE, FAKE, FAKE, FAKE, ws - 16, None) == WS
    g = lib.dhsa_route_topk_csr
    #          Q     K     B  Hq Hkv  L  hd  off   n_ch Nmax k  Qp    Kp    sel   n_sel rp    ci    cost  ws    bytes
    assert g(FAKE, FAKE, 1, 4, 2, 64, 128, FAKE, FAKE, 8, 2, FAKE, FAKE, FAKE, FAKE, None, FAKE, None, FAKE, ws,
             None) == INV
    assert g(FAKE, FAKE, 1, 4, 2, 64, 128, FAKE, FAKE, 8, 2, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, None, FAKE, ws - 16,
             None) == WS


def test_score_topk_csr_arguments_rejected_on_host(lib):
    INV, WS = 1, 5
    f = lib.dhsa_chunk_score_topk_csr
    ws = lib.dhsa_score_topk_workspace_size(1, 4, 8)
    #          Qp    Kp    B  Hq Hkv Nmax off   n_ch  k  sel   n_sel rp    ci    cost  ws    bytes stream
    assert f(FAKE, FAKE, 1, 4, 2, 8, None, FAKE, 2, FAKE, FAKE, FAKE, FAKE, None, FAKE, ws, None) == INV
    assert f(FAKE, FAKE, 1, 4, 2, 8, FAKE, FAKE, 2, FAKE, FAKE, None, FAKE, None, FAKE, ws, None) == INV
    assert f(FAKE, FAKE, 1, 4, 2, 8, FAKE, FAKE, -1, FAKE, FAKE, FAKE, FAKE, None, FAKE, ws, None) == INV
    assert f(FAKE, FAKE, 1, 3, 2, 8, FAKE, FAKE, 2, FAKE, FAKE, FAKE, FAKE, None, FAKE, ws, None) == INV
    assert f(FAKE, FAKE, 1, 4, 2, 8, FAKE, FAKE, 2, FAKE, FAKE, FAKE, FAKE, None, FAKE, ws - 16, None) == WS
    assert f(FAKE, FAKE, 1, 4, 2, 8, FAKE, FAKE, 2, FAKE, FAKE, FAKE, FAKE, None, None, ws, None) == WS


def test_wait_timeout_hook_arguments(lib):
    # host-side only: arming records state for the next launch; bad values are refused
    assert lib.dhsa_debug_arm_wait_timeout(3, 1000) == 1
    assert lib.dhsa_debug_arm_wait_timeout(1, 0) == 1
    assert lib.dhsa_debug_arm_wait_timeout(2, 10 ** 9) == 1
    assert lib.dhsa_debug_arm_wait_timeout(1, 50_000) == 0
    assert lib.dhsa_debug_arm_wait_timeout(0, 0) == 0
