// Token keep-set as a block CSR (stage 4 of the DHSA routing).
//
// OpenReview abstract of "Long-Context Modeling with Dynamic Hierarchical
// Sparse Attention": the chunk-level scores are upsampled to the token level
// to decide which token interactions are kept. Because an upsampled score is
// constant over a chunk, keeping tokens by score keeps whole selected chunks;
// with the causal constraint (gist.science technical summary, Step 2) query
// token t of chunk i keeps key token s iff chunk(s) is selected for i and
// s <= t. That set is represented implicitly by the offsets plus a CSR whose
// row (b, hq, i) lists the kept key chunks in ascending order.
//
// Two launches: a single-CTA exclusive scan of the per-row counts into
// row_ptr (coalesced, four counts per thread per step), then one warp per row
// copying the row's chunk list and computing its cost n_i * sum_j n_j (a
// work estimate for scheduling).
#include "common.cuh"

namespace dhsa {
namespace {

constexpr int kScanThreads = 1024;

// A count outside [0, stride] (a malformed selection) is clamped into it
// here and in fill_rows_kernel alike, so the CSR never outgrows
// dhsa_csr_nnz_upper; fill_rows_kernel flags the row.
__device__ __forceinline__ int row_count(const int32_t* n_sel, long long r, int stride) {
  return min(max(n_sel[r], 0), stride);
}

__global__ void __launch_bounds__(kScanThreads) scan_rows_kernel(const int32_t* __restrict__ n_sel, long long R,
                                                                 int stride, int32_t* __restrict__ row_ptr) {
  // exclusive scan in blocks of 4 * kScanThreads rows: each thread reads four
  // consecutive counts (coalesced across the block), scans them, and the
  // block scans the thread totals; a running carry links the blocks
  __shared__ long long warp_tot[32];
  __shared__ long long carry_s;
  const int t = threadIdx.x, lane = t & 31, warp = t >> 5;
  if (t == 0) carry_s = 0;
  __syncthreads();
  constexpr long long kChunk = 4LL * kScanThreads;
  for (long long base = 0; base < R; base += kChunk) {
    const long long r0 = base + 4LL * t;
    int v[4];
#pragma unroll
    for (int q = 0; q < 4; ++q) v[q] = (r0 + q < R) ? row_count(n_sel, r0 + q, stride) : 0;
    const long long local = (long long)v[0] + v[1] + v[2] + v[3];
    long long incl = local;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const long long u = __shfl_up_sync(0xffffffffu, incl, o);
      if (lane >= o) incl += u;
    }
    if (lane == 31) warp_tot[warp] = incl;
    __syncthreads();
    if (warp == 0) {
      const long long w = warp_tot[lane];
      long long wi = w;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const long long u = __shfl_up_sync(0xffffffffu, wi, o);
        if (lane >= o) wi += u;
      }
      warp_tot[lane] = wi - w;  // exclusive prefix of the warp totals
    }
    __syncthreads();
    const long long carry = carry_s;
    long long run = carry + warp_tot[warp] + incl - local;
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      if (r0 + q < R) row_ptr[r0 + q] = (int32_t)run;
      run += v[q];
    }
    __syncthreads();                                   // everyone has read carry_s
    if (t == kScanThreads - 1) carry_s = run;          // the last thread ends at the block total
    __syncthreads();
  }
  if (t == 0) row_ptr[R] = (int32_t)carry_s;
}

__global__ void __launch_bounds__(256) fill_rows_kernel(const int32_t* __restrict__ sel,
                                                        const int32_t* __restrict__ n_sel, int Hq, int Nmax,
                                                        int stride, const int32_t* __restrict__ off,
                                                        const int32_t* __restrict__ n_chunks,
                                                        const int32_t* __restrict__ row_ptr,
                                                        int32_t* __restrict__ col_idx, int64_t* __restrict__ cost,
                                                        long long R, unsigned int* status) {
  const long long r = ((long long)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  if (r >= R) return;
  const int i = (int)(r % Nmax);
  const int b = (int)(r / ((long long)Hq * Nmax));
  const int32_t* ob = off + (long long)b * (Nmax + 1);
  const int cnt = row_count(n_sel, r, stride);
  const int32_t* src = sel + r * stride;
  int32_t* dst = col_idx + row_ptr[r];
  const int n = min(max(n_chunks[b], 0), Nmax);   // a count outside [0, Nmax] is clamped
  long long keys = 0;
  bool bad = cnt != n_sel[r];
  for (int q = lane; q < cnt; q += 32) {
    const int j = src[q];
    if (j < 0 || j > i || i >= n) {
      bad = true;
      dst[q] = min(max(j, 0), i);   // stored in range, flagged
    } else {
      dst[q] = j;
      keys += ob[j + 1] - ob[j];
    }
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) keys += __shfl_xor_sync(0xffffffffu, keys, o);
  if (__any_sync(0xffffffffu, bad) && lane == 0) raise_device_flag(status, DHSA_DEVFLAG_BAD_SELECTION);
  if (cost && lane == 0) cost[r] = (i < n) ? (long long)(ob[i + 1] - ob[i]) * keys : 0;
}

}  // namespace

int score_topk_stride(int k, int Nmax);

int launch_build_csr(const int32_t* sel, const int32_t* n_sel, int B, int Hq, int Nmax, int k, const int32_t* off,
                     const int32_t* n_chunks, int32_t* row_ptr, int32_t* col_idx, int64_t* cost,
                     unsigned int* status, cudaStream_t stream) {
  const long long R = (long long)B * Hq * Nmax;
  scan_rows_kernel<<<1, kScanThreads, 0, stream>>>(n_sel, R, score_topk_stride(k, Nmax), row_ptr);
  int st = launch_status();
  if (st != DHSA_OK) return st;
  const int threads = 256;
  const long long blocks = (R * 32 + threads - 1) / threads;
  fill_rows_kernel<<<(unsigned)blocks, threads, 0, stream>>>(sel, n_sel, Hq, Nmax, score_topk_stride(k, Nmax), off,
                                                              n_chunks, row_ptr, col_idx, cost, R, status);
  return launch_status();
}

}  // namespace dhsa
