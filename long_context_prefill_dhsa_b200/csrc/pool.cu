// Length-normalised chunk pooling (stage 1 of the DHSA routing).
//
// OpenReview abstract of "Long-Context Modeling with Dynamic Hierarchical
// Sparse Attention": each chunk is represented by the average of its token
// embeddings scaled by the square root of the chunk size, i.e.
//   Xp[b,h,c,:] = sum_{t in chunk c} X[b,h,t,:] / sqrt(n_c).
//
// HBM-bound streaming read of X. One warp owns one (b, h, chunk): lanes 0-15
// read the even rows and lanes 16-31 the odd rows of the chunk, each lane
// 16 bytes (8 bf16) of the 256-byte row, so a warp instruction moves two full
// rows; eight rows per lane are in flight per iteration. The two half-warp
// partial sums are combined with one shuffle, and the 1/sqrt(n) scale is
// applied on the way out. Warps of one block cover consecutive chunks of the
// same head, so a block reads a contiguous span of X.
#include "common.cuh"
#include "pool_row.cuh"

namespace dhsa {
namespace {

__global__ void __launch_bounds__(256) chunk_pool_kernel(const uint4* __restrict__ X, int H, int L,
                                                         const int32_t* __restrict__ off,
                                                         const int32_t* __restrict__ n_chunks, int Nmax,
                                                         long long n_rows, float* __restrict__ Xp,
                                                         unsigned int* status) {
  const long long warp = ((long long)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  if (warp < n_rows) pool_row(X, H, L, off, n_chunks, Nmax, warp, Xp, status);
}

// Q and K in one launch: warps [0, rows_q) pool Q, the rest pool K, so the
// two streams share one grid (no second launch, no tail of a small K grid).
__global__ void __launch_bounds__(256) chunk_pool_qk_kernel(const uint4* __restrict__ Q, const uint4* __restrict__ K,
                                                            int Hq, int Hkv, int L, const int32_t* __restrict__ off,
                                                            const int32_t* __restrict__ n_chunks, int Nmax,
                                                            long long rows_q, long long rows_k,
                                                            float* __restrict__ Qp, float* __restrict__ Kp,
                                                            unsigned int* status) {
  const long long warp = ((long long)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  if (warp < rows_q) pool_row(Q, Hq, L, off, n_chunks, Nmax, warp, Qp, status);
  else if (warp < rows_q + rows_k) pool_row(K, Hkv, L, off, n_chunks, Nmax, warp - rows_q, Kp, status);
}

__global__ void validate_offsets_kernel(const int32_t* __restrict__ off, const int32_t* __restrict__ n_chunks,
                                        int B, int Nmax, int L, unsigned int* status) {
  const long long idx = (long long)blockIdx.x * blockDim.x + threadIdx.x;
  if (idx >= (long long)B * (Nmax + 1)) return;
  const int b = (int)(idx / (Nmax + 1));
  const int c = (int)(idx % (Nmax + 1));
  const int n = n_chunks[b];
  const int32_t* ob = off + (long long)b * (Nmax + 1);
  bool bad = (n < 1 || n > Nmax);
  if (!bad) {
    if (c == 0) bad = ob[0] != 0;
    else if (c < n) bad = !(ob[c] > ob[c - 1] && ob[c] < L);
    else if (c == n) bad = !(ob[c] == L && ob[c] > ob[c - 1]);
    else bad = ob[c] != L;
  }
  if (bad) raise_device_flag(status, DHSA_DEVFLAG_BAD_OFFSETS);
}

}  // namespace

int launch_chunk_pool(const void* X, int B, int H, int L, const int32_t* off, const int32_t* n_chunks, int Nmax,
                      float* Xp, unsigned int* status, cudaStream_t stream) {
  const long long n_rows = (long long)B * H * Nmax;
  const int threads = 256;
  const long long blocks = (n_rows * 32 + threads - 1) / threads;
  chunk_pool_kernel<<<(unsigned)blocks, threads, 0, stream>>>(static_cast<const uint4*>(X), H, L, off, n_chunks,
                                                               Nmax, n_rows, Xp, status);
  return launch_status();
}

int launch_chunk_pool_qk(const void* Q, const void* K, int B, int Hq, int Hkv, int L, const int32_t* off,
                         const int32_t* n_chunks, int Nmax, float* Qp, float* Kp, unsigned int* status,
                         cudaStream_t stream) {
  const long long rows_q = (long long)B * Hq * Nmax, rows_k = (long long)B * Hkv * Nmax;
  const int threads = 256;
  const long long blocks = ((rows_q + rows_k) * 32 + threads - 1) / threads;
  chunk_pool_qk_kernel<<<(unsigned)blocks, threads, 0, stream>>>(static_cast<const uint4*>(Q),
                                                                  static_cast<const uint4*>(K), Hq, Hkv, L, off,
                                                                  n_chunks, Nmax, rows_q, rows_k, Qp, Kp, status);
  return launch_status();
}

int launch_validate_offsets(const int32_t* off, const int32_t* n_chunks, int B, int Nmax, int L,
                            unsigned int* status, cudaStream_t stream) {
  const long long n = (long long)B * (Nmax + 1);
  const int threads = 256;
  validate_offsets_kernel<<<(unsigned)((n + threads - 1) / threads), threads, 0, stream>>>(off, n_chunks, B, Nmax,
                                                                                            L, status);
  return launch_status();
}

}  // namespace dhsa
