/*
 * dhsa.h -- C ABI of the DHSA prefill hot path on NVIDIA B200 (sm_100a).
 *
 * Dynamic Hierarchical Sparse Attention ("Long-Context Modeling with Dynamic
 * Hierarchical Sparse Attention for Memory-Constrained LLM Inference") routes
 * attention hierarchically: the sequence is cut into variable-length chunks,
 * each chunk of Q and K is pooled into one length-normalised vector, the
 * pooled vectors are scored chunk-to-chunk, each query chunk keeps its
 * diagonal chunk plus the top-k earlier chunks, and the chunk decision is
 * expanded to a token keep-set that a causal sparse attention kernel reads.
 * The four calls below are those four stages, in order.
 *
 * Conventions shared by every call
 * --------------------------------
 * - All tensor pointers are DEVICE pointers owned by the caller. The library
 *   never allocates, frees or synchronises; scratch memory is passed in as a
 *   `workspace` whose size is given by the matching *_workspace_size query.
 * - Every compute call is asynchronous on `stream` (a cudaStream_t, passed as
 *   void*; NULL = the legacy default stream). Host-side argument checks run
 *   before anything is enqueued; a call that returns an error enqueued nothing.
 * - Tensors are dense and row-major:
 *     Q   bf16  [B, Hq,  L, head_dim]
 *     K,V bf16  [B, Hkv, L, head_dim]      (GQA: query head hq reads kv head hq / (Hq/Hkv))
 *     off int32 [B, Nmax+1]   chunk c of batch b = tokens [off[b][c], off[b][c+1]);
 *                             off[b][0] = 0, strictly increasing up to
 *                             off[b][n_chunks[b]] = L, padded with L after.
 *     n_chunks int32 [B]      1 <= n_chunks[b] <= Nmax.
 *   One chunk layout per batch element is shared by all heads and by Q/K/V.
 * - head_dim must be 128 (the pages' kernel contract: "BF16, causal,
 *   forward-only, head dimension 128", DHSA README, "Installation").
 * - Return value: a dhsa_status_t. DHSA_ERR_CUDA keeps the CUDA error code
 *   for dhsa_last_cuda_error(). Device-side failures (a bounded wait that
 *   timed out, an offsets table found inconsistent) set a device status word
 *   that dhsa_check_device_status() reads; compute calls never trap.
 * - The library holds no per-call state; calls on different streams may run
 *   concurrently as long as their buffers do not overlap.
 */
#ifndef DHSA_H_
#define DHSA_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  DHSA_OK = 0,
  DHSA_ERR_INVALID_ARG = 1,  /* null pointer, non-positive size, Hq % Hkv != 0, k < 0, Nmax > L, ... */
  DHSA_ERR_UNSUPPORTED = 2,  /* head_dim != 128, or the current device is not sm_100 */
  DHSA_ERR_CUDA = 3,         /* a CUDA runtime call or launch failed; see dhsa_last_cuda_error() */
  DHSA_ERR_DEVICE = 4,       /* a kernel reported an error on the device (dhsa_check_device_status) */
  DHSA_ERR_WORKSPACE = 5     /* workspace pointer null or smaller than the size query asked for */
} dhsa_status_t;

/* Device status word bits, as returned in *device_flags by dhsa_check_device_status. */
#define DHSA_DEVFLAG_WAIT_TIMEOUT 0x1  /* a pipeline wait of the attention kernels or a grid barrier of
                                          the fused routing gave up (that launch's results are undefined) */
#define DHSA_DEVFLAG_BAD_OFFSETS 0x2   /* an inconsistent offsets table: found by dhsa_validate_offsets,
                                          or met (and clamped) by pooling, or met by the attention's
                                          work-list builder (the batch element is then skipped) */
#define DHSA_DEVFLAG_BAD_SELECTION 0x4 /* the CSR builder met a selected chunk outside [0, i] */

/* Human-readable name of a status code (static string, never NULL). */
const char* dhsa_status_string(int status);

/* CUDA error code (cudaError_t as int) of the last DHSA_ERR_CUDA on this host thread. */
int dhsa_last_cuda_error(void);

/* ABI version: major * 10000 + minor * 100 + patch. */
int dhsa_version(void);

/* Synchronises `stream`, reads and clears the current device's status word.
 * Returns DHSA_ERR_DEVICE if any flag was set (flags returned in
 * *device_flags when not NULL), DHSA_ERR_CUDA if the stream itself failed. */
int dhsa_check_device_status(void* stream, uint32_t* device_flags);

/* Checks an offsets table on the device without trusting the host: every
 * batch element must have 1 <= n_chunks[b] <= Nmax, off[b][0] = 0, strictly
 * increasing offsets up to off[b][n_chunks[b]] = L and padding equal to L.
 * A violation sets DHSA_DEVFLAG_BAD_OFFSETS (read it with
 * dhsa_check_device_status). Asynchronous on `stream`. */
int dhsa_validate_offsets(const int32_t* off, const int32_t* n_chunks, int B, int Nmax, int L, void* stream);

/* ---------------------------------------------------------------------------
 * 1. Length-normalised chunk pooling.
 *    Source: OpenReview abstract (chunk representations aggregate the token
 *    embeddings of the chunk; the average is scaled by the square root of the
 *    chunk size) and the gist.science technical summary, "Robust Chunk
 *    Representation".
 *
 *    Xp[b,h,c,:] = (sum over tokens t of chunk c of X[b,h,t,:]) / sqrt(n_c)
 *
 *    X   bf16  [B, H, L, head_dim]  (call once with Q, H = Hq; once with K, H = Hkv)
 *    Xp  fp32  [B, H, Nmax, head_dim], written in full: rows c >= n_chunks[b]
 *        are set to zero. Sums are accumulated in fp32.
 *    A chunk count outside [0, Nmax] or a chunk bound outside [0, L] is
 *    clamped before any row is read and sets DHSA_DEVFLAG_BAD_OFFSETS; no
 *    read leaves the head's L rows.
 * ------------------------------------------------------------------------- */
int dhsa_chunk_pool(const void* X, int B, int H, int L, int head_dim, const int32_t* off,
                    const int32_t* n_chunks, int Nmax, float* Xp, void* stream);

/* 1b. Both poolings of a layer in one launch: Qp from Q [B, Hq, L, 128] and
 *     Kp from K [B, Hkv, L, 128], each exactly as dhsa_chunk_pool computes it
 *     (same arithmetic, bit-identical results). Hq % Hkv == 0; all four
 *     pointers 16-byte aligned; errors as for dhsa_chunk_pool. */
int dhsa_chunk_pool_qk(const void* Q, const void* K, int B, int Hq, int Hkv, int L, int head_dim,
                       const int32_t* off, const int32_t* n_chunks, int Nmax, float* Qp, float* Kp, void* stream);

/* ---------------------------------------------------------------------------
 * 2. Chunk similarity and causal per-query-chunk top-k.
 *    Source: gist.science technical summary, "Hierarchical Routing
 *    Formulation", Steps 1-2 (a chunk-level similarity matrix; each query
 *    chunk is routed to a compact set of chunks under the causal constraint).
 *
 *    For each row (b, hq, i < n_chunks[b]):
 *      S[j] = <Qp[b,hq,i,:], Kp[b,hq/G,j,:]> for j < i, ranked as the fp64
 *             dot product of the fp32 inputs (computed in fp32; only scores
 *             within the fp32 rounding bound of the cut are re-scored in
 *             fp64); the diagonal needs no score;
 *      kept = {i} + the min(k, i) earlier chunks ranked by (S descending,
 *             j ascending) -- ties go to the lower chunk index;
 *      sel[b,hq,i, 0 .. n_sel-1] = kept in ascending order (diagonal last),
 *      the rest of the row = -1; n_sel[b,hq,i] = min(k, i) + 1.
 *    Rows i >= n_chunks[b] get n_sel = 0 and are filled with -1.
 *
 *    Qp fp32 [B, Hq, Nmax, 128], Kp fp32 [B, Hkv, Nmax, 128] (as written by 1.)
 *    sel   int32 [B, Hq, Nmax, sel_stride], sel_stride = dhsa_sel_stride(k, Nmax)
 *    n_sel int32 [B, Hq, Nmax]
 *    k >= Nmax - 1 keeps every earlier chunk (dense causal).
 *    workspace: dhsa_score_topk_workspace_size(B, Hq, Nmax) bytes: pooled-key
 *    norms plus the packed fp32 scores (row i keeps its i scores) of a batch
 *    of heads -- all heads when they fit in 256 MiB, else as many as fit
 *    (at least one); the call then loops over head batches.
 * ------------------------------------------------------------------------- */
int dhsa_sel_stride(int k, int Nmax);
size_t dhsa_score_topk_workspace_size(int B, int Hq, int Nmax);
int dhsa_chunk_score_topk(const float* Qp, const float* Kp, int B, int Hq, int Hkv, int Nmax,
                          const int32_t* n_chunks, int k, int32_t* sel, int32_t* n_sel, void* workspace,
                          size_t workspace_bytes, void* stream);

/* ---------------------------------------------------------------------------
 * 2'. Chunk similarity and causal selection under a token budget per row.
 *    Sources: README, "Predictor Checkpoints" (static checkpoints use a fixed
 *    row budget, dynamic ones a query-dependent row budget); gist.science
 *    technical summary, "Significance and Claims" (N_b is the token budget,
 *    cost about O(L * N_b)). The pages give no formula; the rule implemented
 *    (and restated by the test oracle) is:
 *
 *    For each row (b, hq, i < n_chunks[b]), with n_j = off[b][j+1] - off[b][j]:
 *      r      = min(recent, i, k_max)   -- the chunks i-r .. i-1 are always kept
 *      N_b    = budgets ? budgets[b,hq,i] : budget
 *      ranked = the chunks j < i - r by (S descending, j ascending), S as in 2.
 *      walk the ranked chunks in order, keeping each while fewer than
 *      k_max - r have been kept and the kept earlier tokens (recent window
 *      included) are still fewer than N_b;
 *      sel[b,hq,i, ...] = kept ranked chunks, then the window, then i
 *      (ascending), the rest -1; n_sel = their count (<= k_max + 1).
 *    Rows i >= n_chunks[b] get n_sel = 0 and are filled with -1.
 *
 *    off      int32 [B, Nmax+1] as in 1.;  budgets int32 [B, Hq, Nmax] or NULL
 *    budget   >= 0 (used when budgets is NULL);  recent >= 0
 *    k_max    0 .. dhsa_budget_max_chunks() (UNSUPPORTED above it)
 *    sel      int32 [B, Hq, Nmax, dhsa_sel_stride(k_max, Nmax)];  n_sel as in 2.
 *    workspace: dhsa_score_topk_workspace_size(B, Hq, Nmax) bytes.
 *    The CSR of 3. is then built with k = k_max.
 * ------------------------------------------------------------------------- */
int dhsa_budget_max_chunks(void);
int dhsa_chunk_score_select_budget(const float* Qp, const float* Kp, int B, int Hq, int Hkv, int Nmax,
                                   const int32_t* off, const int32_t* n_chunks, int budget,
                                   const int32_t* budgets, int recent, int k_max, int32_t* sel, int32_t* n_sel,
                                   void* workspace, size_t workspace_bytes, void* stream);

/* 2b. Similarity and top-k as in 2., writing the block CSR of 3. as well.
 *    Under the top-k rule row i < n_chunks[b] keeps min(k, i) + 1 chunks, so
 *    every row's CSR offset has a closed form and each selection row writes
 *    its CSR row directly (no scan, no second pass over sel). Results equal
 *    dhsa_chunk_score_topk followed by dhsa_build_block_csr, bit for bit:
 *    sel and n_sel as in 2., row_ptr / col_idx / cost (nullable) as in 3.
 *    (col_idx needs dhsa_csr_nnz_upper(B, Hq, Nmax, k) entries). off is the
 *    offsets table of 1. Workspace and errors as for 2. */
int dhsa_chunk_score_topk_csr(const float* Qp, const float* Kp, int B, int Hq, int Hkv, int Nmax,
                              const int32_t* off, const int32_t* n_chunks, int k, int32_t* sel, int32_t* n_sel,
                              int32_t* row_ptr, int32_t* col_idx, int64_t* cost, void* workspace,
                              size_t workspace_bytes, void* stream);

/* ---------------------------------------------------------------------------
 * 2c. Pooling, similarity and top-k in one launch.
 *    Sources as for 1. and 2.; the gist.science technical summary places the
 *    routing module right after the Q/K projections, so it runs as one unit.
 *
 *    Does what dhsa_chunk_pool_qk followed by dhsa_chunk_score_topk do, with
 *    the same results bit for bit, as one cooperative launch: pooling of Q
 *    and K, key norms and score tiles, then the selection, separated by
 *    grid-wide barriers (each bounded: a block that waits more than 1 s at a
 *    barrier sets DHSA_DEVFLAG_WAIT_TIMEOUT and an abort word, and every
 *    block then leaves the kernel; the outputs of that launch are undefined).
 *    Arguments and layouts are those of the two calls; Qp and Kp are written
 *    as by 1b. On B200 the separate launches are faster (they keep more
 *    warps in flight for the HBM-bound pooling and the latency-bound
 *    selection); this entry serves callers that want one launch.
 *    workspace: dhsa_route_fused_workspace_size(B, Hq, Nmax) bytes (equal to
 *    dhsa_score_topk_workspace_size; its first 8 bytes hold the barrier
 *    count and the abort word, reset by this call on `stream`). Calls
 *    sharing a workspace must not overlap on the GPU.
 * ------------------------------------------------------------------------- */
size_t dhsa_route_fused_workspace_size(int B, int Hq, int Nmax);
int dhsa_route_fused(const void* Q, const void* K, int B, int Hq, int Hkv, int L, int head_dim, const int32_t* off,
                     const int32_t* n_chunks, int Nmax, int k, float* Qp, float* Kp, int32_t* sel, int32_t* n_sel,
                     void* workspace, size_t workspace_bytes, void* stream);

/* 2d. The one launch of 2c. also writing the block CSR of 3., as 2b. does.
 *    Results equal dhsa_route_fused followed by dhsa_build_block_csr, bit
 *    for bit. row_ptr, col_idx and cost (nullable) as in 3.; other
 *    arguments, the workspace and errors as for 2c. */
int dhsa_route_topk_csr(const void* Q, const void* K, int B, int Hq, int Hkv, int L, int head_dim,
                        const int32_t* off, const int32_t* n_chunks, int Nmax, int k, float* Qp, float* Kp,
                        int32_t* sel, int32_t* n_sel, int32_t* row_ptr, int32_t* col_idx, int64_t* cost,
                        void* workspace, size_t workspace_bytes, void* stream);

/* ---------------------------------------------------------------------------
 * 3. Upsampling to the token keep-set, stored as a block CSR.
 *    Source: OpenReview abstract (chunk scores are upsampled to the token
 *    level to decide which token interactions are kept); gist.science
 *    technical summary, Step 2 (high-scoring chunks expand into their tokens
 *    under the causal constraint).
 *
 *    Query token t of chunk i keeps key token s iff chunk(s) is in sel(i) and
 *    s <= t. That set is never materialised: it is the CSR below plus `off`.
 *    Rows r = (b*Hq + hq)*Nmax + i:
 *      row_ptr int32 [B*Hq*Nmax + 1]  exclusive prefix sum of n_sel
 *      col_idx int32 [row_ptr[last]]  kept chunks of row r, ascending (diagonal last)
 *      cost    int64 [B*Hq*Nmax] or NULL: n_i * sum_{j in sel(i)} n_j, 0 for padded rows
 *    col_idx needs room for dhsa_csr_nnz_upper(B, Hq, Nmax, k) entries.
 * ------------------------------------------------------------------------- */
size_t dhsa_csr_nnz_upper(int B, int Hq, int Nmax, int k);
int dhsa_build_block_csr(const int32_t* sel, const int32_t* n_sel, int B, int Hq, int Nmax, int k,
                         const int32_t* off, const int32_t* n_chunks, int32_t* row_ptr, int32_t* col_idx,
                         int64_t* cost, void* stream);

/* ---------------------------------------------------------------------------
 * 4. Causal block-sparse attention forward over the kept chunk pairs.
 *    Source: DHSA README, "Overview" (block-sparse attention extended to
 *    variable-sized query and key blocks) and "Installation" (BF16, causal,
 *    forward-only, head dim 128); gist.science technical summary, "Key
 *    Technical Components" (tiled online-softmax backend that never builds
 *    the full attention matrix).
 *
 *    O[b,hq,t,:] = sum_s softmax_s(scale * <Q[b,hq,t], K[b,hkv,s]>) V[b,hkv,s]
 *    over the kept keys s of token t only (hkv = hq / (Hq/Hkv)); fp32
 *    accumulation and softmax statistics, bf16 output (round to nearest).
 *    The probabilities enter the PV product rounded to bf16; their
 *    exponentials come from the hardware ex2 approximation and, for one pair
 *    in four, from a degree-3 polynomial with relative error <= 1.02e-4 (both
 *    give exactly 0 for a masked key).
 *    Every row of V must be finite, including rows that are not kept (a
 *    masked key contributes 0 * V[s]).
 *
 *    row_ptr / col_idx as written by 3. (cost may be NULL; it is not read yet).
 *    A col_idx entry outside [0, i] is clamped into it (3. flags such rows).
 *    O bf16 [B, Hq, L, 128]; every token row of every head is written, except
 *    in a batch element whose offsets table is inconsistent (that element is
 *    skipped and DHSA_DEVFLAG_BAD_OFFSETS set).
 *    workspace: dhsa_sparse_attn_workspace_size(B, Hq, L, Nmax) bytes.
 * ------------------------------------------------------------------------- */
size_t dhsa_sparse_attn_workspace_size(int B, int Hq, int L, int Nmax);
int dhsa_sparse_attn_fwd(const void* Q, const void* K, const void* V, int B, int Hq, int Hkv, int L,
                         int head_dim, const int32_t* off, const int32_t* n_chunks, int Nmax,
                         const int32_t* row_ptr, const int32_t* col_idx, const int64_t* cost,
                         float softmax_scale, void* O, void* workspace, size_t workspace_bytes, void* stream);

/* ---------------------------------------------------------------------------
 * 4b. The same attention forward without a caller workspace.
 *    The paper has no counterpart: this is a deployment variant of 4.
 *
 *    For callers that cannot call cudaMalloc: code that runs inside an
 *    engine's pre-planned device-memory arena (every byte is reserved up
 *    front, so an extra allocation fails or fragments it), and code on a
 *    latency-critical path where cudaMalloc's implicit device-wide
 *    synchronisation would stall other streams. The work list that 4. keeps
 *    in `workspace` is kept instead in a 4 MiB static device array of the
 *    library (held by every GPU that loads the library until process exit).
 *    Problems whose work list does not fit, i.e.
 *      dhsa_sparse_attn_workspace_size(B, Hq, L, Nmax) > 4 MiB,
 *    are rejected with DHSA_ERR_WORKSPACE before anything is enqueued
 *    (use 4. for those). This call performs no cudaMalloc/cudaFree and calls
 *    no allocating library routine.
 *
 *    The first call on each device looks up the array's device address
 *    (cudaGetSymbolAddress) and caches it; make that first call before any
 *    stream capture. All calls share the one array and it keeps the last
 *    call's contents; nothing in it has to start at zero (each call rewrites
 *    the whole work list and its count). Calls whose executions overlap on
 *    the GPU (other streams, other host threads) race on the array: order
 *    them, e.g. on one stream.
 *
 *    Arguments, layouts and results are those of dhsa_sparse_attn_fwd.
 * ------------------------------------------------------------------------- */
int dhsa_sparse_attn_fwd_noalloc(const void* Q, const void* K, const void* V, int B, int Hq, int Hkv, int L,
                                 int head_dim, const int32_t* off, const int32_t* n_chunks, int Nmax,
                                 const int32_t* row_ptr, const int32_t* col_idx, float softmax_scale, void* O,
                                 void* stream);

/* ---------------------------------------------------------------------------
 * 4c. The same attention forward with a choice of query-tile shapes.
 *    The paper has no counterpart: the DHSA README ("Overview") stresses that
 *    chunks are variable-sized, and a chunk whose last 128-row query tile
 *    holds few rows leaves most of that tile idle. This entry can hand such
 *    rows to a second kernel whose tiles hold at most 64 query rows (keys on
 *    the tensor core's M side, queries on its N side).
 *
 *    short_tiles: 0 = every query tile has 128 rows (this is
 *    dhsa_sparse_attn_fwd); 1 = a chunk's last tile goes to the 64-row kernel
 *    when it holds at most 64 rows; 2 = every chunk is cut into 64-row tiles.
 *    Other values: DHSA_ERR_INVALID_ARG. The output is the same computation
 *    for every choice (the order of the fp32 sums differs, so results may
 *    differ in the last bf16 place). On B200 the 64-row kernel is not faster
 *    per query row than the 128-row one (its two MMAs both stream their
 *    operands from shared memory), so 0 is the fast choice.
 *
 *    workspace: dhsa_sparse_attn_tiles_workspace_size(B, Hq, L, Nmax,
 *    short_tiles) bytes (0 for invalid arguments). Other arguments, layouts,
 *    results and errors as for dhsa_sparse_attn_fwd.
 * ------------------------------------------------------------------------- */
size_t dhsa_sparse_attn_tiles_workspace_size(int B, int Hq, int L, int Nmax, int short_tiles);
int dhsa_sparse_attn_fwd_tiles(const void* Q, const void* K, const void* V, int B, int Hq, int Hkv, int L,
                               int head_dim, const int32_t* off, const int32_t* n_chunks, int Nmax,
                               const int32_t* row_ptr, const int32_t* col_idx, float softmax_scale, int short_tiles,
                               void* O, void* workspace, size_t workspace_bytes, void* stream);

/* ---------------------------------------------------------------------------
 * 5. Test hook of the bounded device waits.
 *    The paper has no counterpart. Every wait of the pipelined kernels gives
 *    up after 1 s and reports DHSA_DEVFLAG_WAIT_TIMEOUT instead of hanging;
 *    this hook lets a test make such a wait run out on purpose, without any
 *    fault, so that the path is exercised:
 *      mode 1: the next attention launch (4., 4b. or 4c. with 128-row tiles)
 *              holds back its scheduler, so the other roles' first wait --
 *              which precedes every copy and MMA -- runs out after limit_ns;
 *              the CTAs record the flag, free their TMEM and return without
 *              writing O.
 *      mode 2: the next one-launch routing (2c., 2d.) has block 0 arrive
 *              late at its first grid barrier; the other blocks give up
 *              after limit_ns, set the abort word, and all blocks leave.
 *      mode 0: disarm.
 *    The hook is one-shot (the launch that uses it disarms it) and host-side
 *    state of the library: not thread-safe, for tests only.
 *    limit_ns: 1 .. 100,000,000 for modes 1 and 2 (DHSA_ERR_INVALID_ARG else).
 * ------------------------------------------------------------------------- */
int dhsa_debug_arm_wait_timeout(int mode, uint64_t limit_ns);

#ifdef __cplusplus
}
#endif

#endif /* DHSA_H_ */
