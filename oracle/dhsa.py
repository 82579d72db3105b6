"""CPU oracle for the DHSA prefill path -- TEST INFRASTRUCTURE ONLY.

Plain, slow, obviously-correct NumPy restatement of what the path computes.
Only the tests, the package's smoke check and the benchmark's CPU-baseline leg
may import it; the product path never does. It shares no code with the CUDA
library: inputs arrive as arrays (bf16 as uint16 bit patterns) and every step
is written out from its definition in float64 (attention may run in float32
for large workloads, as the caller asks).

Sources (the pages on DHSA, "Long-Context Modeling with Dynamic Hierarchical
Sparse Attention for Memory-Constrained LLM Inference"):

* pool    -- OpenReview abstract: chunk representations aggregate the token
             embeddings of each chunk, and the average is scaled by the square
             root of the chunk size; the gist.science technical summary,
             "Robust Chunk Representation", says the same (sum divided by the
             true chunk length, then a length normalisation).
* scores  -- gist.science technical summary, "Hierarchical Routing
             Formulation", Step 1: a chunk-level similarity matrix estimates
             the importance of chunk-to-chunk interactions.
* select  -- same, Step 2: each query chunk is routed to a compact set of
             key chunks under the causal constraint; the kept set is the
             diagonal chunk plus the top-k earlier chunks, ties to the lower
             chunk index.
* upsample/attention -- OpenReview abstract (chunk scores upsampled to the
             token level decide which token interactions are kept) and the
             README, "Installation": the kernel is causal, forward-only, BF16,
             head dimension 128.

Parity pins: every function here is pinned by tests under tests/ to values
fixed independently of this file (hand-computed pooling cases, a brute-force
token-level block score, dense causal attention written separately, and
invariants). Two parts stay "parity unpinned": real predictor boundaries and
real row budgets (the trained weights do not exist here), so offsets, k and
the token budgets are inputs. The row-budget rule itself is a reading of the
pages (they name the budget but fix no formula); its pins check it against
the top-k rule it reduces to and against closed forms.
"""
from __future__ import annotations

import math

import numpy as np

HEAD_DIM = 128


# ---------------------------------------------------------------- helpers
def bf16_to_f64(u16: np.ndarray) -> np.ndarray:
    """Exact upcast of bf16 bit patterns (uint16) to float64."""
    return (np.asarray(u16).astype(np.uint32) << 16).view(np.float32).astype(np.float64)


def chunk_bounds(off_b: np.ndarray, c: int):
    return int(off_b[c]), int(off_b[c + 1])


# ---------------------------------------------------------------- a1: pooling
def chunk_pool(X: np.ndarray, off: np.ndarray, n_chunks: np.ndarray, nmax: int) -> np.ndarray:
    """Length-normalised chunk pooling (OpenReview abstract).

    Xp[b,h,c,:] = mean(X[b,h,rows of c,:]) * sqrt(n_c) = sum(rows) / sqrt(n_c).
    X is float64 [B,H,L,d]; rows c >= n_chunks[b] of the result are zero.
    """
    B, H, L, d = X.shape
    Xp = np.zeros((B, H, nmax, d), dtype=np.float64)
    for b in range(B):
        for c in range(int(n_chunks[b])):
            s, e = chunk_bounds(off[b], c)
            n = e - s
            Xp[b, :, c, :] = X[b, :, s:e, :].mean(axis=1) * math.sqrt(n)
    return Xp


# ---------------------------------------------------------------- a2: similarity
def chunk_scores(Qp: np.ndarray, Kp: np.ndarray, n_chunks: np.ndarray) -> np.ndarray:
    """Chunk similarity S[b,hq,i,j] = <Qp[b,hq,i], Kp[b,hq//G,j]> for j < i.

    Raw dot product of the pooled vectors (the pages name a similarity matrix
    without a formula; a positive scale would not change any ranking).
    Entries with j >= i, or outside the batch element's chunks, are NaN.
    """
    B, Hq, nmax, d = Qp.shape
    Hkv = Kp.shape[1]
    G = Hq // Hkv
    S = np.full((B, Hq, nmax, nmax), np.nan)
    for b in range(B):
        n = int(n_chunks[b])
        for hq in range(Hq):
            full = Qp[b, hq, :n] @ Kp[b, hq // G, :n].T
            ii, jj = np.tril_indices(n, -1)
            S[b, hq, ii, jj] = full[ii, jj]
    return S


# ---------------------------------------------------------------- a3: top-k
def select_row(S_row: np.ndarray, i: int, k: int) -> np.ndarray:
    """Kept chunks of query chunk i: {i} + the top-k of j < i.

    Order: score descending, ties to the lower j (a stable sort of -S over
    ascending j). With i <= k every earlier chunk is kept. Returned ascending,
    so the diagonal chunk i comes last.
    """
    cand = np.arange(i)
    order = cand[np.argsort(-S_row[:i], kind="stable")]
    keep = np.sort(order[: min(k, i)])
    return np.concatenate([keep, [i]]).astype(np.int64)


def select(S: np.ndarray, n_chunks: np.ndarray, k: int):
    """sel[b][hq][i] -> ascending int array of kept key chunks."""
    B, Hq = S.shape[:2]
    return [[[select_row(S[b, hq, i], i, k) for i in range(int(n_chunks[b]))]
             for hq in range(Hq)] for b in range(B)]


def tie_gap(S_row: np.ndarray, i: int, k: int) -> float:
    """Score gap between the k-th and (k+1)-th earlier chunk in selection order
    (inf when i <= k: nothing is cut)."""
    if i <= k:
        return math.inf
    srt = np.sort(S_row[:i])[::-1]
    return float(srt[k - 1] - srt[k]) if k > 0 else math.inf


def near_tie(S_row: np.ndarray, i: int, k: int, rel: float = 1e-5) -> bool:
    """A row is a near-tie when its cut gap is below rel * max_j |S[i, j]|."""
    if i <= k or k == 0:
        return False
    scale = float(np.max(np.abs(S_row[:i])))
    return tie_gap(S_row, i, k) < rel * scale


# ---------------------------------------------------------------- a3': row budgets
# README, "Predictor Checkpoints": static checkpoints use a fixed row budget,
# dynamic ones a query-dependent row budget. gist.science technical summary,
# "Significance and Claims" (Scalability): N_b is the token budget and the
# per-layer cost is about O(L * N_b). The codewithpapers record names
# recent-key-block and row-budget helpers but shows no code. Reading taken
# (the pages fix no formula): a row keeps its diagonal chunk, the `recent`
# chunks just before it, and then earlier chunks in rank order (score
# descending, ties to the lower index) while the kept earlier tokens are
# still fewer than the budget, at most k_max earlier chunks in all.
def select_budget_row(S_row: np.ndarray, lens: np.ndarray, i: int, budget: int, recent: int,
                      k_max: int) -> np.ndarray:
    """Kept chunks of query chunk i under a token budget; ascending, i last.

    lens[j] is the token length of chunk j. The recent window is the last
    r = min(recent, i, k_max) chunks before i; ranked chunks are the j < i - r.
    """
    r = min(recent, i, k_max)
    recent_js = list(range(i - r, i))
    used = int(sum(int(lens[j]) for j in recent_js))
    cand = np.arange(i - r)
    order = cand[np.argsort(-S_row[: i - r], kind="stable")]
    taken = []
    for j in order:
        if len(taken) + r >= k_max or used >= budget:
            break
        taken.append(int(j))
        used += int(lens[j])
    keep = sorted(taken) + recent_js
    return np.array(keep + [i], dtype=np.int64)


def select_budget(S: np.ndarray, off: np.ndarray, n_chunks: np.ndarray, budget, recent: int, k_max: int):
    """sel[b][hq][i] under a token budget: an int for every row, or an int
    array [B, Hq, Nmax] of per-row budgets."""
    B, Hq = S.shape[:2]
    out = []
    for b in range(B):
        n = int(n_chunks[b])
        lens = np.diff(off[b][: n + 1])
        rows_b = []
        for hq in range(Hq):
            rows_b.append([select_budget_row(S[b, hq, i], lens, i,
                                             int(budget if np.isscalar(budget) else budget[b, hq, i]),
                                             recent, k_max) for i in range(n)])
        out.append(rows_b)
    return out


def budget_near_tie(S_row: np.ndarray, lens: np.ndarray, i: int, budget: int, recent: int, k_max: int,
                    rel: float = 1e-5) -> bool:
    """The kept set can change under a swap of two ranked chunks whose scores
    differ by less than rel * max_j |S[i, j]| (j over every earlier chunk,
    window included) anywhere in the ranked prefix the rule inspects.

    The walk takes ranks 0 .. t-1 in order (t = chunks it took) and stops
    without looking at rank t's identity, so the adjacent pairs that decide
    the set are (0,1), ..., (t-1,t) -- the taken chunks and the next one.
    """
    r = min(recent, i, k_max)
    c = i - r
    if c < 2:
        return False
    kept = select_budget_row(S_row, lens, i, budget, recent, k_max)
    t = len(kept) - 1 - r                # ranked chunks taken
    last = min(t + 1, c)                 # ranks 0 .. last-1 decide the set
    if last < 2:
        return False
    srt = np.sort(S_row[:c])[::-1]
    scale = float(np.max(np.abs(S_row[:i])))
    gaps = srt[: last - 1] - srt[1:last]
    return bool(gaps.min() < rel * scale)


# ---------------------------------------------------------------- a4: CSR
def block_csr(sel, off: np.ndarray, n_chunks: np.ndarray, nmax: int):
    """Block CSR of kept key chunks, one row per (b, hq, query chunk).

    Rows are ordered (b, hq, i) with i < nmax; padded rows (i >= N_b) are
    empty. cost = n_i * sum_{j in sel} n_j (int64).
    """
    B, Hq = len(sel), len(sel[0])
    row_ptr = [0]
    cols, cost = [], []
    for b in range(B):
        n = int(n_chunks[b])
        lens = np.diff(off[b, : n + 1]).astype(np.int64)
        for hq in range(Hq):
            for i in range(nmax):
                if i < n:
                    s = sel[b][hq][i]
                    cols.extend(int(j) for j in s)
                    cost.append(int(lens[i]) * int(lens[s].sum()))
                else:
                    cost.append(0)
                row_ptr.append(len(cols))
    return (np.array(row_ptr, dtype=np.int64), np.array(cols, dtype=np.int64),
            np.array(cost, dtype=np.int64))


def token_keep_mask(sel_bh, off_b: np.ndarray, n: int, L: int) -> np.ndarray:
    """Token keep-set of one (b, hq) as an explicit L x L boolean matrix.

    Query token t in chunk i keeps key token s iff chunk(s) is kept for i and
    s <= t (the upsampling of the chunk decision to token level with the
    causal constraint). For small L only.
    """
    M = np.zeros((L, L), dtype=bool)
    for i in range(n):
        qs, qe = chunk_bounds(off_b, i)
        for j in sel_bh[i]:
            ks, ke = chunk_bounds(off_b, int(j))
            M[qs:qe, ks:ke] = True
    return M & np.tril(np.ones((L, L), dtype=bool))


# ---------------------------------------------------------------- a5: attention
def attn_chunk(Q, K, V, off_b, kept, i, scale, dtype=np.float64):
    """Output rows of query chunk i for one (b, hq): softmax over kept keys only.

    Q: [L,d] of the query head, K/V: [L,d] of its kv head. Keys are the union
    of the kept chunks' rows, in ascending order; inside the diagonal chunk
    key s is visible to query t iff s <= t.
    """
    qs, qe = chunk_bounds(off_b, i)
    rows = np.concatenate([np.arange(*chunk_bounds(off_b, int(j))) for j in kept])
    q = Q[qs:qe].astype(dtype)
    k = K[rows].astype(dtype)
    v = V[rows].astype(dtype)
    logits = (q @ k.T) * dtype(scale)
    t = np.arange(qs, qe)[:, None]
    logits = np.where(rows[None, :] <= t, logits, -np.inf)
    m = logits.max(axis=1, keepdims=True)
    p = np.exp(logits - m)
    return (p @ v) / p.sum(axis=1, keepdims=True)


def attn_sparse(Q, K, V, off, n_chunks, sel, scale=None, dtype=np.float64,
                rows=None):
    """Sparse causal attention over the kept chunk pairs.

    Q [B,Hq,L,d], K/V [B,Hkv,L,d] as float arrays. Returns O [B,Hq,L,d]
    (dtype). `rows` optionally restricts the work to a list of (b, hq, i);
    other rows of O are left as NaN.
    """
    B, Hq, L, d = Q.shape
    G = Hq // K.shape[1]
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    O = np.full((B, Hq, L, d), np.nan, dtype=dtype)
    todo = rows if rows is not None else [
        (b, hq, i) for b in range(B) for hq in range(Hq) for i in range(int(n_chunks[b]))]
    for (b, hq, i) in todo:
        qs, qe = chunk_bounds(off[b], i)
        O[b, hq, qs:qe] = attn_chunk(Q[b, hq], K[b, hq // G], V[b, hq // G], off[b],
                                     sel[b][hq][i], i, scale, dtype)
    return O


def attn_dense(Q, K, V, scale=None, dtype=np.float64):
    """Textbook dense causal softmax attention with GQA (no chunks)."""
    B, Hq, L, d = Q.shape
    G = Hq // K.shape[1]
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    O = np.empty((B, Hq, L, d), dtype=dtype)
    causal = np.tril(np.ones((L, L), dtype=bool))
    for b in range(B):
        for hq in range(Hq):
            q = Q[b, hq].astype(dtype)
            k = K[b, hq // G].astype(dtype)
            v = V[b, hq // G].astype(dtype)
            s = np.where(causal, (q @ k.T) * dtype(scale), -np.inf)
            s = s - s.max(axis=1, keepdims=True)
            p = np.exp(s)
            O[b, hq] = (p / p.sum(axis=1, keepdims=True)) @ v
    return O


# ---------------------------------------------------------------- whole path
def kept_pairs(off, n_chunks, sel):
    """Kept token pairs per (b, hq): sum_i n_i * sum_{j in sel, j<i} n_j + n_i(n_i+1)/2."""
    B, Hq = len(sel), len(sel[0])
    out = np.zeros((B, Hq), dtype=np.int64)
    for b in range(B):
        n = int(n_chunks[b])
        lens = np.diff(off[b, : n + 1]).astype(np.int64)
        for hq in range(Hq):
            tot = 0
            for i in range(n):
                s = sel[b][hq][i]
                tot += int(lens[i]) * int(lens[s[:-1]].sum()) + int(lens[i]) * (int(lens[i]) + 1) // 2
            out[b, hq] = tot
    return out


def density(off, n_chunks, sel, L):
    """Kept token pairs / causal pairs L(L+1)/2, averaged over (b, hq)."""
    return float(kept_pairs(off, n_chunks, sel).mean() / (L * (L + 1) / 2))


def routing(Q, K, off, n_chunks, k):
    """Pool -> score -> select for float64 Q [B,Hq,L,d], K [B,Hkv,L,d]."""
    nmax = off.shape[1] - 1
    Qp = chunk_pool(Q, off, n_chunks, nmax)
    Kp = chunk_pool(K, off, n_chunks, nmax)
    S = chunk_scores(Qp, Kp, n_chunks)
    return Qp, Kp, S, select(S, n_chunks, k)
