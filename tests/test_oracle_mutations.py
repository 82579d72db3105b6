"""The oracle's pins catch plausible mistakes.

Each case swaps one function of the oracle (on the CPU, for the duration of
the case) for a version with a typical slip -- a wrong normalisation, a
dropped or extra term, a flipped tie rule, a shifted mask, a wrong head map
-- and checks that at least one of the pins in test_oracle_pins.py then
fails. Nothing here touches the CUDA library.
"""
import math

import numpy as np
import pytest

from oracle import dhsa
from tests import test_oracle_pins as pins

_PINS = [
    (pins.test_pool_hand_cases, {}),
    (pins.test_pool_concat_two_equal_chunks, {}),
    (pins.test_pool_padded_rows_zero_and_multi_batch, {}),
    (pins.test_select_matches_bruteforce_block_mask, {"c": 4, "m": 12, "k": 3, "G": 1}),
    (pins.test_select_matches_bruteforce_block_mask, {"c": 5, "m": 16, "k": 5, "G": 4}),
    (pins.test_select_ties_go_to_lower_index, {}),
    (pins.test_select_edges, {}),
    (pins.test_csr_by_hand, {}),
    (pins.test_kept_pairs_by_hand, {}),
    (pins.test_attn_k_all_equals_dense, {}),
    (pins.test_attn_k0_is_per_chunk_causal, {}),
    (pins.test_attn_matches_explicit_token_mask, {}),
    (pins.test_attn_single_token_and_convexity, {}),
    (pins.test_budget_hand_cases, {}),
    (pins.test_budget_reduces_to_topk, {"seed": 0}),
    (pins.test_budget_uniform_lengths_is_topk_of_budget_over_length, {}),
    (pins.test_budget_zero_keeps_recent_window_only, {}),
    (pins.test_budget_invariants_random, {}),
    (pins.test_budget_near_tie_hand_cases, {}),
    (pins.test_density_by_hand, {}),
    (pins.test_bf16_upcast_bit_patterns, {}),
]


def _failing_pins():
    failed = []
    for fn, kw in _PINS:
        try:
            fn(**kw)
        except Exception:          # an assertion or an error the slip provokes
            failed.append(fn.__name__)
    return failed


# ------------------------------------------------------------ the slips
def _pool_mean(X, off, n_chunks, nmax):
    """Mean instead of mean * sqrt(n)."""
    P = _orig["chunk_pool"](X, off, n_chunks, nmax)
    out = P.copy()
    for b in range(off.shape[0]):
        for c in range(int(n_chunks[b])):
            out[b, :, c] = P[b, :, c] / math.sqrt(int(off[b, c + 1] - off[b, c]))
    return out


def _pool_sum(X, off, n_chunks, nmax):
    """Plain sum: the 1/sqrt(n) dropped."""
    P = _orig["chunk_pool"](X, off, n_chunks, nmax)
    out = P.copy()
    for b in range(off.shape[0]):
        for c in range(int(n_chunks[b])):
            out[b, :, c] = P[b, :, c] * math.sqrt(int(off[b, c + 1] - off[b, c]))
    return out


def _scores_wrong_group(Qp, Kp, n_chunks):
    """Query head hq scored against kv head hq % Hkv instead of hq // G."""
    B, Hq, nmax, _ = Qp.shape
    Hkv = Kp.shape[1]
    Kr = Kp[:, [h % Hkv for h in range(Hq)]]
    S = np.zeros((B, Hq, nmax, nmax))
    for b in range(B):
        S[b] = np.einsum("hid,hjd->hij", Qp[b], Kr[b])
    mask = np.tril(np.ones((nmax, nmax), dtype=bool), k=-1)
    return np.where(mask[None, None], S, 0.0)


def _select_ties_high(S_row, i, k):
    """Ties to the higher chunk index."""
    cand = np.arange(i)[::-1]
    order = cand[np.argsort(-S_row[:i][::-1], kind="stable")]
    keep = np.sort(order[: min(k, i)])
    return np.concatenate([keep, [i]]).astype(np.int64)


def _select_one_more(S_row, i, k):
    """k + 1 earlier chunks."""
    return _orig["select_row"](S_row, i, k + 1)


def _select_no_diag(S_row, i, k):
    """The diagonal chunk left out when there are earlier chunks."""
    r = _orig["select_row"](S_row, i, k)
    return r[:-1] if len(r) > 1 else r


def _attn_scale_sq(Q, K, V, off_b, kept, i, scale, dtype=np.float64):
    """Scores scaled by 1/d instead of 1/sqrt(d)."""
    return _orig["attn_chunk"](Q, K, V, off_b, kept, i, scale * scale, dtype)


def _attn_strict_causal(Q, K, V, off_b, kept, i, scale, dtype=np.float64):
    """Key s visible to query t only if s < t (a token no longer sees itself)."""
    qs, qe = dhsa.chunk_bounds(off_b, i)
    rows = np.concatenate([np.arange(*dhsa.chunk_bounds(off_b, int(j))) for j in kept])
    q, k, v = Q[qs:qe].astype(dtype), K[rows].astype(dtype), V[rows].astype(dtype)
    logits = (q @ k.T) * dtype(scale)
    t = np.arange(qs, qe)[:, None]
    logits = np.where(rows[None, :] < t, logits, -np.inf)
    m = np.max(np.where(np.isfinite(logits), logits, -1e300), axis=1, keepdims=True)
    p = np.where(np.isfinite(logits), np.exp(logits - m), 0.0)
    den = p.sum(axis=1, keepdims=True)
    return (p @ v) / np.where(den > 0, den, 1.0)


def _budget_strict(S_row, lens, i, budget, recent, k_max):
    """Stops only once the kept tokens exceed the budget (> instead of >=)."""
    return _orig["select_budget_row"](S_row, lens, i, budget + 1, recent, k_max)


def _budget_window_uncounted(S_row, lens, i, budget, recent, k_max):
    """The recent window's tokens not counted against the budget."""
    r = min(recent, i, k_max)
    extra = int(sum(int(lens[j]) for j in range(i - r, i)))
    return _orig["select_budget_row"](S_row, lens, i, budget + extra, recent, k_max)


def _near_tie_signed_scale(S_row, lens, i, budget, recent, k_max, rel=1e-5):
    """Band relative to max S instead of max |S|."""
    r = min(recent, i, k_max)
    c = i - r
    t = len(dhsa.select_budget_row(S_row, lens, i, budget, recent, k_max)) - 1 - r
    last = min(t + 1, c)
    if c < 2 or last < 2:
        return False
    srt = np.sort(S_row[:c])[::-1]
    return bool(np.min(srt[: last - 1] - srt[1:last]) < rel * float(np.max(S_row[:i])))


def _near_tie_past_boundary(S_row, lens, i, budget, recent, k_max, rel=1e-5):
    """Also counts the pair just past the boundary (ranks t and t+1)."""
    if _orig["budget_near_tie"](S_row, lens, i, budget, recent, k_max, rel):
        return True
    r = min(recent, i, k_max)
    c = i - r
    t = len(dhsa.select_budget_row(S_row, lens, i, budget, recent, k_max)) - 1 - r
    srt = np.sort(S_row[:c])[::-1]
    scale = float(np.max(np.abs(S_row[:i])))
    return bool(t + 1 < c and srt[t] - srt[t + 1] < rel * scale)


def _near_tie_no_boundary(S_row, lens, i, budget, recent, k_max, rel=1e-5):
    """Only gaps between taken chunks; the (last taken, next) pair dropped."""
    r = min(recent, i, k_max)
    c = i - r
    t = len(dhsa.select_budget_row(S_row, lens, i, budget, recent, k_max)) - 1 - r
    if t < 2:
        return False
    srt = np.sort(S_row[:c])[::-1]
    scale = float(np.max(np.abs(S_row[:i])))
    return bool(np.min(srt[: t - 1] - srt[1:t]) < rel * scale)


def _near_tie_window_ignored(S_row, lens, i, budget, recent, k_max, rel=1e-5):
    """Ranks taken over every earlier chunk, window chunks included."""
    return _orig["budget_near_tie"](S_row, lens, i, budget, 0, k_max, rel)


def _near_tie_scale_without_window(S_row, lens, i, budget, recent, k_max, rel=1e-5):
    """Scale from the ranked candidates only (the window's scores left out)."""
    r = min(recent, i, k_max)
    s = np.array(S_row, dtype=np.float64)
    if r > 0:
        s[i - r:i] = 0.0
    return _orig["budget_near_tie"](s, lens, i, budget, recent, k_max, rel)


def _density_half_square(off, n_chunks, sel, L):
    """Causal pairs taken as L^2 / 2."""
    return float(dhsa.kept_pairs(off, n_chunks, sel).mean() / (L * L / 2))


def _density_strict_causal(off, n_chunks, sel, L):
    """Causal pairs taken as L(L-1)/2 (the diagonal left out)."""
    return float(dhsa.kept_pairs(off, n_chunks, sel).mean() / (L * (L - 1) / 2))


def _density_summed(off, n_chunks, sel, L):
    """Heads summed instead of averaged."""
    return float(dhsa.kept_pairs(off, n_chunks, sel).sum() / (L * (L + 1) / 2))


def _bf16_as_f16(u16):
    """Bit patterns read as IEEE half precision."""
    return np.asarray(u16).astype(np.uint16).view(np.float16).astype(np.float64)


def _bf16_short_shift(u16):
    """Shifted by 15 instead of 16."""
    return (np.asarray(u16).astype(np.uint32) << 15).view(np.float32).astype(np.float64)


_orig = {name: getattr(dhsa, name) for name in
         ("chunk_pool", "chunk_scores", "select_row", "attn_chunk", "select_budget_row", "budget_near_tie",
          "density", "bf16_to_f64")}

SLIPS = [
    ("chunk_pool", _pool_mean),
    ("chunk_pool", _pool_sum),
    ("chunk_scores", _scores_wrong_group),
    ("select_row", _select_ties_high),
    ("select_row", _select_one_more),
    ("select_row", _select_no_diag),
    ("attn_chunk", _attn_scale_sq),
    ("attn_chunk", _attn_strict_causal),
    ("select_budget_row", _budget_strict),
    ("select_budget_row", _budget_window_uncounted),
    ("budget_near_tie", _near_tie_signed_scale),
    ("budget_near_tie", _near_tie_past_boundary),
    ("budget_near_tie", _near_tie_no_boundary),
    ("budget_near_tie", _near_tie_window_ignored),
    ("budget_near_tie", _near_tie_scale_without_window),
    ("density", _density_half_square),
    ("density", _density_strict_causal),
    ("density", _density_summed),
    ("bf16_to_f64", _bf16_as_f16),
    ("bf16_to_f64", _bf16_short_shift),
]


def test_pins_pass_on_the_oracle_as_written():
    assert _failing_pins() == []


@pytest.mark.parametrize("name,slip", SLIPS, ids=[s[1].__name__ for s in SLIPS])
def test_a_slip_fails_some_pin(monkeypatch, name, slip):
    monkeypatch.setattr(dhsa, name, slip)
    failed = _failing_pins()
    assert failed, f"no pin caught {slip.__name__}: {slip.__doc__}"
